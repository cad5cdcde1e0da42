// attn.cu -- step 3 of the decode path: exact softmax attention over the
// selected K/V rows, as split-K flash decoding followed by a combine.
//
// HyLRA sec. 2.3: tolerant layers attend over a subset of the KV cache given by
// top-k indices (possibly an earlier layer's); DSA stage 2 in "Flash Attention
// vs Sparse Attention": full attention over the selected tokens only.  The
// online softmax (running max and sum, rescaled per tile) is the same page's
// "tiling + online softmax"; it gives the same result as the two-pass softmax.
// A null index list means every valid row (a full-attention layer, as the
// Flux Attention router or a HyLRA sensitive layer chooses).
//
// Design: grid = (split, unit); a CTA is 8 warps and owns a contiguous range of
// the unit's index list, walked in tiles of 128 rows (16 per warp).  Two ways
// of bringing a tile's K and V (256 B a row) into shared memory:
//   - gather (an index list of tokens): each warp fetches its own 16 rows with
//     16-byte vector loads (a half-warp per row) one tile ahead in registers,
//     or, when the CTA's range is a single tile, with cp.async straight into
//     shared memory (no registers held, so two CTAs fit an SM); rows are padded
//     to 272 B so the fragment loads below are free of bank conflicts, and no
//     barrier wider than a warp is needed per tile.  (One TMA bulk copy per
//     256-byte row was the first design: issuing them cost ~13 ns a copy.)
//   - contiguous tiles (full attention, or a 128-token block): four 2-D TMA
//     tensor loads a tile in the 128-byte swizzle into a 3-stage ring, each
//     stage completing on an mbarrier, refilled as soon as it is consumed.
// Each warp then runs, on its
// 16 rows, the two contractions of flash decoding on the tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate), with the g <= 8 query heads as
// the M dimension padded to 16:
//   S = Q K^T   (8 k-steps, K fragments by ldmatrix),
//   online softmax per head on the S fragments (fp32, log2 units),
//   O += P V    (P split as bf16 hi + bf16 lo so that the weights keep ~16
//               bits; V fragments by ldmatrix.trans).
// tcgen05's smallest M is 64, so there 87-94% of every MMA would be padding;
// the m16 warp MMA fits a GQA group.  The 8 warps are merged at the end into
// the CTA's partial (M, L, acc[128]) per head.  When a unit has at most 8
// splits and every unit's cluster can be resident at once, the splits of a unit
// form one thread-block cluster: each CTA pushes the slices of its partial to
// the CTAs that own those output slices (posted distributed-shared-memory
// stores), one cluster barrier, and each CTA combines its slice locally (no
// scratch).  Otherwise (more splits, or more clusters than fit: a B200 holds
// only 15 clusters of 8 CTAs of ~226 KB) each CTA writes its partial to the
// workspace and the last CTA of the unit to arrive (an atomic counter in the
// workspace, reset by that CTA) combines the partials into O.
#include <cooperative_groups.h>
#include <cstring>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace tsa {

constexpr int kMaxSplits = 256;
constexpr int kClusterMax = 8;  // splits per unit that combine inside one (portable) cluster
constexpr int kSms = 148;
constexpr int kPartStride = kD + 4;  // M, L, 2 pad, acc[128]: 528 B, 16-byte aligned
constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = 8;
constexpr int kTileRows = 128;                         // 16 rows per warp
constexpr int kRowStride = kD * 2 + 16;                // 272 B: padded so 8 rows hit 8 bank groups
constexpr int kStageBytes = kTileRows * kRowStride * 2;  // K and V of one tile: 68 KB
constexpr int kRing = 3;                               // tiles in flight (the multi-tile kernel)
constexpr long kWaitSpins = 1L << 22;                  // bounded mbarrier wait (then flag + go on)

template <int G>
struct AttnCfg {
    static constexpr int kPer = G * 16;  // output float4 slots per CTA when S >= 2
    static constexpr int kRecvBytes = kClusterMax * kPer * 16;
    static constexpr int kAccBytes = kAttnWarps * G * kD * 4;
    static constexpr int work_bytes(int stages) {
        return stages * kStageBytes > kAccBytes ? stages * kStageBytes : kAccBytes;
    }
    static constexpr int smem_bytes(int stages, bool cluster) {
        return 1024 /* alignment slack */ + work_bytes(stages) + (cluster ? kRecvBytes : 0);
    }
};

__device__ __forceinline__ unsigned smem_u32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// Wait for the phase with the given parity; gives up after kWaitSpins polls,
// raising the timeout flag (the copies are still bounded: they read valid rows).
__device__ __forceinline__ void mbar_wait(uint64_t* bar, unsigned parity, unsigned* flag) {
    const unsigned a = smem_u32(bar);
    for (long i = 0; i < kWaitSpins; ++i) {
        unsigned done;
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
                     : "=r"(done) : "r"(a), "r"(parity) : "memory");
        if (done) return;
    }
    atomicOr(flag, kFlagTimeout);
}
// 1-D bulk copy (TMA engine) global -> this CTA's shared memory, completing on `bar`
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void ldsm_x4(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.  Only the rows of A that
// carry query heads (a0/a1 and a4/a5: row lane/4) are non-zero here, so the
// rows lane/4 + 8 of A are passed as zero.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
// byte offset of 16-byte chunk `chunk` of row `row` in a tile of padded rows
__device__ __forceinline__ int roff(int row, int chunk) { return row * kRowStride + (chunk << 4); }

// CONTIG: every tile is 128 consecutive cache rows (a full-attention range, or
// one 128-token block in block mode) and arrives by 2-D TMA tensor loads in the
// 128-byte-swizzled layout (4 loads per tile); otherwise each row is its own
// 256-byte bulk copy into rows padded to 272 bytes.
// ONE (gather only): every CTA's range is one tile; rows are copied straight into
// shared memory (cp.async) instead of through registers, so two CTAs fit an SM.
template <int G, int STAGES, bool CLUSTER, bool CONTIG, bool ONE>
__global__ void __launch_bounds__(kAttnThreads, ONE ? 2 : 1)
attn_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
            const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
            const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ lens,
            const int32_t* __restrict__ idx, const int32_t* __restrict__ kreq, int k_max,
            int block, int Hkv, int Ncap, float scale_log2, int S, float* __restrict__ part,
            unsigned* __restrict__ counters, float* __restrict__ O, unsigned* __restrict__ flag, int early,
            float* __restrict__ sout, float scale, float* __restrict__ lse) {
    using Cfg = AttnCfg<G>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // 1024-byte aligned work area (the swizzled layout needs it)
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ float s_wm[kAttnWarps][G], s_wl[kAttnWarps][G];
    __shared__ float s_M[G], s_L[G];
    __shared__ float s_Mr[kClusterMax][G], s_Lr[kClusterMax][G];  // cluster path: received (M, L)
    __shared__ int s_last;
    __shared__ __align__(8) uint64_t s_bar[STAGES];
    __shared__ int s_first[STAGES];  // CONTIG: first cache row of the tile in each stage, or -1

    const int s = blockIdx.x, unit = blockIdx.y;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;  // mma fragment coordinates
    // early: the kernel before this one did not write the lengths, the k's or Q
    // (the decode step's own top-k), so they are read before waiting on it
    int len = 0, kreq_b = k_max;
    if (early) {
        len = lens[b];
        if (kreq) kreq_b = kreq[b];
    }
    griddep_wait();
    griddep_launch();
    if (!early) {
        len = lens[b];
        if (kreq) kreq_b = kreq[b];
    }
    if (len < 0 || len > Ncap) {
        if (tid == 0 && s == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    int npos, nb = 0;
    if (idx == nullptr) {
        npos = len;
    } else {
        nb = block == 1 ? len : ceil_div(len, block);
        int kb = max(0, min(kreq_b, nb));
        if (kb > k_max) {
            if (tid == 0 && s == 0) atomicOr(flag, kFlagBounds);
            kb = k_max;
        }
        npos = kb * block;
    }
    const int chunk = CONTIG ? ceil_div(ceil_div(npos, S), kTileRows) * kTileRows : ceil_div(npos, S);
    const int p0 = min(s * chunk, npos), p1 = min(p0 + chunk, npos);
    const int ntiles = ceil_div(p1 - p0, kTileRows);
    const int32_t* iu = idx ? idx + (size_t)unit * k_max : nullptr;
    const __nv_bfloat16* Ku = K + (size_t)unit * Ncap * kD;
    const __nv_bfloat16* Vu = V + (size_t)unit * Ncap * kD;

    // cache row of position pos, or -1 (skipped entry, tail of a partial block)
    auto row_of = [&](int pos) -> int {
        if (iu == nullptr) return pos;
        if (block == 1) {
            const int r = iu[pos];
            if (r >= len) {
                atomicOr(flag, kFlagBounds);
                return -1;
            }
            return r < 0 ? -1 : r;
        }
        const int slot = pos / block;
        const int e = iu[slot];
        if (e >= nb) {
            atomicOr(flag, kFlagBounds);
            return -1;
        }
        if (e < 0) return -1;
        const int r = e * block + (pos - slot * block);
        return r < len ? r : -1;
    };
    // CONTIG: the tile's first cache row (dense: its position; block mode: the
    // chosen block's first row), or -1 when the block entry is absent
    auto tile_first = [&](int t) -> int {
        const int pos0 = p0 + t * kTileRows;
        if (t >= ntiles) return -1;
        if (iu == nullptr) return pos0;
        const int e = iu[pos0 / kTileRows];
        if (e >= nb) {
            atomicOr(flag, kFlagBounds);
            return -1;
        }
        return e < 0 ? -1 : e * kTileRows;
    };
    // thread 0 issues the tile's four tensor loads (K and V, two 64-dim halves
    // each); `first` was read ahead of time so the index latency stays hidden
    auto stage_contig = [&](int t, int first) {
        if (t >= ntiles) return;
        const int st = t % STAGES;
        s_first[st] = first;
        if (first >= 0) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&s_bar[st], 4 * 64 * kTileRows * 2);
            const unsigned dst = smem_u32(smem + st * kStageBytes);
            const unsigned bar = smem_u32(&s_bar[st]);
            const int y = unit * Ncap + first;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
                        dst + h * 64 * kTileRows * 2),
                    "l"(&kmap), "r"(h * 64), "r"(y), "r"(bar)
                    : "memory");
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
                        dst + 2 * 64 * kTileRows * 2 + h * 64 * kTileRows * 2),
                    "l"(&vmap), "r"(h * 64), "r"(y), "r"(bar)
                    : "memory");
            }
        } else {
            mbar_arrive(&s_bar[st]);
        }
    };
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < STAGES; ++i) mbar_init(&s_bar[i], CONTIG ? 1 : kTileRows);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    // CONTIG: the first STAGES tiles' block indices in one round, then their loads
    int next_first = -1;  // CONTIG, thread 0: first row of the tile that refills the stage next
    if constexpr (CONTIG) {
        if (tid == 0) {
            int f[STAGES];
#pragma unroll
            for (int t = 0; t < STAGES; ++t) f[t] = tile_first(t);
#pragma unroll
            for (int t = 0; t < STAGES; ++t) stage_contig(t, f[t]);
        }
    }

    const int r0 = warp * 16;  // this warp's rows in a tile
    // Gather: each warp fetches its own 16 rows of a tile with 16-byte vector
    // loads (a half-warp per 256-byte row; lane l takes chunk l & 15 of rows
    // (l >> 4), +2, ..., +14), one tile ahead in registers, and stores them
    // into its rows of the padded tile: no TMA queue (one 256-byte bulk copy
    // per row issued at ~13 ns a copy per SM, which bounded short gathers) and
    // no CTA barrier per tile.  Rows not in the set are zeros (0 x NaN = NaN).
    unsigned char* kw = smem + r0 * kRowStride;
    unsigned char* vw = smem + (kTileRows + r0) * kRowStride;
    const int hl = lane >> 4, c16 = lane & 15;
    uint4 pk[8], pv[8];
    uint32_t vm_next = 0;
    auto fetch = [&](int t) {
        if constexpr (CONTIG) return;
        int myrow = -1;
        if (lane < 16) {
            const int pos = p0 + t * kTileRows + r0 + lane;
            if (pos < p1) myrow = row_of(pos);
        }
        vm_next = __ballot_sync(0xffffffffu, myrow >= 0) & 0xffffu;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int rr = __shfl_sync(0xffffffffu, myrow, hl + 2 * j);
            pk[j] = rr >= 0 ? ld_stream(Ku + (size_t)rr * kD + 8 * c16) : make_uint4(0, 0, 0, 0);
            pv[j] = rr >= 0 ? ld_stream(Vu + (size_t)rr * kD + 8 * c16) : make_uint4(0, 0, 0, 0);
        }
    };
    // ONE: cp.async copies of tile t's rows of this warp (zeros for rows not in the set)
    uint32_t vm_one = 0;
    auto issue_one = [&](int t) {
        int myrow = -1;
        if (lane < 16) {
            const int pos = p0 + t * kTileRows + r0 + lane;
            if (pos < p1) myrow = row_of(pos);
        }
        vm_one = __ballot_sync(0xffffffffu, myrow >= 0) & 0xffffu;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int rr = __shfl_sync(0xffffffffu, myrow, hl + 2 * j);
            unsigned char* kd = kw + (hl + 2 * j) * kRowStride + 16 * c16;
            unsigned char* vd = vw + (hl + 2 * j) * kRowStride + 16 * c16;
            if (rr >= 0) {
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(kd)),
                             "l"(Ku + (size_t)rr * kD + 8 * c16) : "memory");
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(vd)),
                             "l"(Vu + (size_t)rr * kD + 8 * c16) : "memory");
            } else {
                *reinterpret_cast<uint4*>(kd) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
            }
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    if constexpr (!CONTIG) {
        if (ntiles > 0) {  // in flight while Q is read
            if constexpr (ONE) issue_one(0);
            else fetch(0);
        }
    }

    // A fragments of Q (bf16, unscaled: the scale is applied to S in fp32).
    // Row g of A = query head g of the group (zero for g >= G); rows g+8 are zero.
    uint32_t qa[8][2];
    {
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(Q + ((size_t)unit * G + (g < G ? g : 0)) * kD);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qa[ks][0] = g < G ? qrow[ks * 8 + t4] : 0u;       // dims 16ks + 2t4, +1
            qa[ks][1] = g < G ? qrow[ks * 8 + 4 + t4] : 0u;   // dims 16ks + 8 + 2t4, +1
        }
    }
    float o[16][4];  // O fragments: head g, dims 8n + 2t4 (+1); [2],[3] are padding rows
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // this warp's running max / sum for head g

    const unsigned sbase = smem_u32(smem);
    // The two contractions of flash decoding on this warp's 16 rows of a tile
    // (K at kt, V at vt); bit i of vm: row r0 + i is in the set.
    // sout (full attention that also emits its top-k, contiguous tiles only): the
    // scores of the tile's rows -- scale x the max over the group's heads of q.k,
    // the criterion a SELECT layer scores by -- written as S is formed
    float* const su_out = (CONTIG && sout) ? sout + (size_t)unit * Ncap : nullptr;
    auto warp_tile = [&](unsigned kt, unsigned vt, uint32_t vm, int first) {
        // byte offset of 16-byte chunk c of tile row r (padded rows, or the
        // 128-byte swizzle of the TMA tensor loads: two 64-dim halves)
        auto off = [&](int r, int c) -> unsigned {
            if constexpr (CONTIG)
                return (unsigned)((c >> 3) * 64 * kTileRows * 2 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
            else
                return (unsigned)roff(r, c);
        };
        // ---- S = Q K^T over this warp's 16 rows (two n-tiles of 8 rows)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int m = lane >> 3, i = lane & 7;  // ldmatrix: matrix m, row i
            const int row = r0 + (m >> 1) * 8 + i;   // n-tile (m>>1), k-half (m&1)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kt + off(row, 2 * ks + (m & 1)), b0, b1, b2, b3);
                mma_bf16(sc[0], qa[ks][0], qa[ks][1], b0, b1);
                mma_bf16(sc[1], qa[ks][0], qa[ks][1], b2, b3);
            }
        }
        if constexpr (CONTIG) {
            if (su_out) {  // uniform: the max over heads g < G of each row's dot, by lanes of equal t4
                float e[4] = {g < G ? sc[0][0] : -INFINITY, g < G ? sc[0][1] : -INFINITY,
                              g < G ? sc[1][0] : -INFINITY, g < G ? sc[1][1] : -INFINITY};
#pragma unroll
                for (int o = 4; o < 32; o <<= 1)
#pragma unroll
                    for (int q = 0; q < 4; ++q) e[q] = fmaxf(e[q], __shfl_xor_sync(0xffffffffu, e[q], o));
                if (g == 0) {
                    const int ia = 2 * t4;
                    const int lrow[4] = {ia, ia + 1, ia + 8, ia + 9};
#pragma unroll
                    for (int q = 0; q < 4; ++q)  // scale > 0: scale x max = max of the scaled logits
                        if ((vm >> lrow[q]) & 1u) su_out[first + r0 + lrow[q]] = e[q] * scale;
                }
            }
        }
        // ---- online softmax for head g (columns = rows of the tile)
        float z[4];
        {
            const int ia = 2 * t4;  // local rows of sc[0][0..1]; sc[1] adds 8
            z[0] = (vm >> ia) & 1u ? sc[0][0] * scale_log2 : -INFINITY;
            z[1] = (vm >> (ia + 1)) & 1u ? sc[0][1] * scale_log2 : -INFINITY;
            z[2] = (vm >> (ia + 8)) & 1u ? sc[1][0] * scale_log2 : -INFINITY;
            z[3] = (vm >> (ia + 9)) & 1u ? sc[1][1] * scale_log2 : -INFINITY;
        }
        float mt = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        const float mnew = fmaxf(m_run, mt);
        if (mnew != -INFINITY) {  // uniform across the 4 lanes of head g
            const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - mnew);
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) p[e] = z[e] == -INFINITY ? 0.f : exp2f(z[e] - mnew);
            float ps = (p[0] + p[1]) + (p[2] + p[3]);
            ps += __shfl_xor_sync(0xffffffffu, ps, 1);
            ps += __shfl_xor_sync(0xffffffffu, ps, 2);
            l_run = l_run * alpha + ps;
            m_run = mnew;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                o[n][0] *= alpha;
                o[n][1] *= alpha;
            }
            // P as the A operand (row g, k = tile rows), split hi + lo
            const uint32_t ph0 = pack_bf16(p[0], p[1]), ph1 = pack_bf16(p[2], p[3]);
            const __nv_bfloat162 h0 = *reinterpret_cast<const __nv_bfloat162*>(&ph0);
            const __nv_bfloat162 h1 = *reinterpret_cast<const __nv_bfloat162*>(&ph1);
            const uint32_t pl0 = pack_bf16(p[0] - __low2float(h0), p[1] - __high2float(h0));
            const uint32_t pl1 = pack_bf16(p[2] - __low2float(h1), p[3] - __high2float(h1));
            // ---- O += P V over 16 dim n-tiles
            const int m = lane >> 3, i = lane & 7;  // ldmatrix.trans: matrix m, row i
            const int row = r0 + (m & 1) * 8 + i;    // k-half (m&1), dim n-tile (m>>1)
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vt + off(row, 2 * np + (m >> 1)), b0, b1, b2, b3);
                mma_bf16(o[2 * np], ph0, ph1, b0, b1);
                mma_bf16(o[2 * np], pl0, pl1, b0, b1);
                mma_bf16(o[2 * np + 1], ph0, ph1, b2, b3);
                mma_bf16(o[2 * np + 1], pl0, pl1, b2, b3);
            }
        }
    };

    if constexpr (CONTIG) {
        for (int t = 0; t < ntiles; ++t) {
            if (tid == 0) next_first = tile_first(t + STAGES);  // in flight during this tile
            mbar_wait(&s_bar[t % STAGES], (unsigned)(t / STAGES) & 1u, flag);  // tile t has landed
            const int st = t % STAGES;
            // the valid rows are a prefix: the range's and the sequence's ends cut it;
            // an absent block (first < 0) has none and nothing landed
            const int first = s_first[st];
            int tile_rows = min(kTileRows, p1 - p0 - t * kTileRows);
            tile_rows = first < 0 ? 0 : max(0, min(tile_rows, len - first));
            // rows past it hold real cache data, which may be anything: give V
            // there zeros, since their weight 0 times NaN is NaN
            const bool zero = tile_rows > 0 && tid >= tile_rows && tid < kTileRows;
            if (zero) {
                unsigned char* vrow = smem + st * kStageBytes + 2 * 64 * kTileRows * 2 + tid * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4*>(vrow + h * 64 * kTileRows * 2 + 16 * c) = make_uint4(0, 0, 0, 0);
                fence_proxy_async();  // before the stage's next tensor load overwrites them
            }
            __syncthreads();  // every thread, every tile (never a divergent barrier)
            const int nv = tile_rows - r0;
            const uint32_t vm = nv >= 16 ? 0xffffu : (nv > 0 ? (1u << nv) - 1u : 0u);
            if (vm) {  // warp-uniform
                const unsigned kt = sbase + st * kStageBytes;
                warp_tile(kt, kt + 2 * 64 * kTileRows * 2, vm, first);
            }
            __syncthreads();  // every warp is done with this stage
            if (tid == 0) stage_contig(t + STAGES, next_first);  // refill it (nothing past the end)
        }
    } else if constexpr (ONE) {
        for (int t = 0; t < ntiles; ++t) {  // one tile (any count stays correct, unpipelined)
            if (t > 0) issue_one(t);
            asm volatile("cp.async.wait_all;\n" ::: "memory");
            __syncwarp();
            if (vm_one) warp_tile(sbase, sbase + kTileRows * kRowStride, vm_one, 0);
            __syncwarp();  // the math has read these rows before the next copies land
        }
    } else {
        for (int t = 0; t < ntiles; ++t) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                *reinterpret_cast<uint4*>(kw + (hl + 2 * j) * kRowStride + 16 * c16) = pk[j];
                *reinterpret_cast<uint4*>(vw + (hl + 2 * j) * kRowStride + 16 * c16) = pv[j];
            }
            const uint32_t vm = vm_next;
            __syncwarp();
            if (t + 1 < ntiles) fetch(t + 1);  // the next tile's loads fly during this tile's math
            if (vm) warp_tile(sbase, sbase + kTileRows * kRowStride, vm, 0);
            __syncwarp();  // the math has read these rows before the next store
        }
    }
    __syncthreads();

    // ---- merge the 4 warps: each warp's (m, l, o) for heads g < G
    float* s_acc = reinterpret_cast<float*>(smem);  // [kAttnWarps][G][128], over the staging ring
    if (g < G) {
#pragma unroll
        for (int n = 0; n < 16; ++n)
            *reinterpret_cast<float2*>(s_acc + (warp * G + g) * kD + 8 * n + 2 * t4) = make_float2(o[n][0], o[n][1]);
        if (t4 == 0) {
            s_wm[warp][g] = m_run;
            s_wl[warp][g] = l_run;
        }
    }
    __syncthreads();
    if (tid < G) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_wm[w][tid]);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w)
            L += s_wm[w][tid] == -INFINITY ? 0.f : s_wl[w][tid] * exp2f(s_wm[w][tid] - M);
        s_M[tid] = M;
        s_L[tid] = L;
    }
    __syncthreads();
    const int nslots = G * 32;  // (head, quad of dims) output slots: thread tid owns slot tid
    const bool has_slot = tid < nslots;
    const int h_me = tid >> 5, qd_me = tid & 31;
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    if (has_slot) {
        const float M = s_M[h_me];
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            const float wm = s_wm[w][h_me];
            const float sc = (wm == -INFINITY || M == -INFINITY) ? 0.f : exp2f(wm - M);
            const float4 a = *reinterpret_cast<const float4*>(s_acc + (w * G + h_me) * kD + 4 * qd_me);
            A.x += a.x * sc;
            A.y += a.y * sc;
            A.z += a.z * sc;
            A.w += a.w * sc;
        }
    }

    if constexpr (CLUSTER) {
        if (S == 1) {  // nothing to combine
            if (has_slot) {
                const float L = s_L[h_me];
                float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
                if (L > 0.f) r = make_float4(A.x / L, A.y / L, A.z / L, A.w / L);
                *reinterpret_cast<float4*>(O + ((size_t)unit * G + h_me) * kD + 4 * qd_me) = r;
                if (lse && qd_me == 0) lse[(size_t)unit * G + h_me] = L > 0.f ? s_M[h_me] + log2f(L) : -INFINITY;
            }
            return;
        }
        // the S splits of this unit are the S CTAs of this cluster (rank = split)
        cg::cluster_group cluster = cg::this_cluster();
        const int per = ceil_div(nslots, S);  // output slots owned by each CTA
        float4* recv = reinterpret_cast<float4*>(smem + Cfg::work_bytes(STAGES));  // [src][Cfg::kPer]
        if (has_slot) {
            const int owner = tid / per, lslot = tid - owner * per;
            *cluster.map_shared_rank(recv + s * Cfg::kPer + lslot, owner) = A;
        }
        if (tid < G * S) {
            const int r = tid / G, h = tid - (tid / G) * G;
            *cluster.map_shared_rank(&s_Mr[s][h], r) = s_M[h];
            *cluster.map_shared_rank(&s_Lr[s][h], r) = s_L[h];
        }
        cluster.sync();  // every slice has arrived at its owner
        for (int ls = tid; ls < per; ls += kAttnThreads) {
            const int slot = s * per + ls;
            if (slot >= nslots) break;
            const int h = slot >> 5, qd = slot & 31;
            float M = -INFINITY;
            for (int j = 0; j < S; ++j) M = fmaxf(M, s_Mr[j][h]);
            float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
            float den = 0.f;
            if (M != -INFINITY) {
                for (int j = 0; j < S; ++j) {
                    const float w = s_Mr[j][h] == -INFINITY ? 0.f : exp2f(s_Mr[j][h] - M);
                    const float4 oj = recv[j * Cfg::kPer + ls];
                    den += w * s_Lr[j][h];
                    num.x += w * oj.x;
                    num.y += w * oj.y;
                    num.z += w * oj.z;
                    num.w += w * oj.w;
                }
            }
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
            if (den > 0.f) r = make_float4(num.x / den, num.y / den, num.z / den, num.w / den);
            *reinterpret_cast<float4*>(O + ((size_t)unit * G + h) * kD + 4 * qd) = r;
            if (lse && qd == 0) lse[(size_t)unit * G + h] = den > 0.f ? M + log2f(den) : -INFINITY;
        }
        return;  // no remote access after the barrier: CTAs may leave in any order
    } else {
        if (has_slot) {
            float* pu = part + (((size_t)unit * S + s) * G + h_me) * kPartStride;
            *reinterpret_cast<float4*>(pu + 4 + 4 * qd_me) = A;
            if (qd_me == 0) *reinterpret_cast<float2*>(pu) = make_float2(s_M[h_me], s_L[h_me]);
        }
        // the last CTA of this unit to arrive combines all splits
        __threadfence();
        __syncthreads();
        if (tid == 0) s_last = atomicAdd(&counters[unit], 1u) == (unsigned)(S - 1);
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        float* s_cm = reinterpret_cast<float*>(smem);  // [S*G], over the staging ring
        float* s_cl = s_cm + kMaxSplits * G;
        const float* pall = part + (size_t)unit * S * G * kPartStride;
        for (int i = tid; i < S * G; i += kAttnThreads) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(pall + (size_t)i * kPartStride));
            s_cm[i] = ml.x;
            s_cl[i] = ml.y;
        }
        __syncthreads();
        for (int slot = tid; slot < nslots; slot += kAttnThreads) {
            const int h = slot >> 5, qd = slot & 31;
            float M = -INFINITY;
            for (int j = 0; j < S; ++j) M = fmaxf(M, s_cm[j * G + h]);
            float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
            float den = 0.f;
            if (M != -INFINITY) {
#pragma unroll 8
                for (int j = 0; j < S; ++j) {
                    const float mj = s_cm[j * G + h];
                    const float w = mj == -INFINITY ? 0.f : exp2f(mj - M);
                    const float4 oj = __ldcg(reinterpret_cast<const float4*>(pall + ((size_t)j * G + h) * kPartStride + 4 + 4 * qd));
                    den += w * s_cl[j * G + h];
                    num.x += w * oj.x;
                    num.y += w * oj.y;
                    num.z += w * oj.z;
                    num.w += w * oj.w;
                }
            }
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
            if (den > 0.f) r = make_float4(num.x / den, num.y / den, num.z / den, num.w / den);
            *reinterpret_cast<float4*>(O + ((size_t)unit * G + h) * kD + 4 * qd) = r;
            if (lse && qd == 0) lse[(size_t)unit * G + h] = den > 0.f ? M + log2f(den) : -INFINITY;
        }
        if (tid == 0) counters[unit] = 0u;  // ready for the next launch on this workspace
    }
}

int attn_splits(const Dims& d, int k_max, int block, bool dense) {
    const int units = d.units() > 0 ? d.units() : 1;
    long long rows;
    int s;
    if (dense) {
        // bandwidth-bound streaming at one CTA per SM: the split count that
        // minimises (waves) x (tiles per CTA + ~2 tiles of fixed cost), so no
        // second wave runs a handful of CTAs alone; past 8 splits the partials
        // combine through the workspace (small next to the stream)
        rows = d.Ncap;
        const long long tiles = (rows + kTileRows - 1) / kTileRows;
        long long best = -1;
        s = 1;
        for (int c = 1; c <= kMaxSplits && c <= tiles; ++c) {
            const long long waves = ((long long)units * c + kSms - 1) / kSms;
            const long long cost = waves * ((tiles + c - 1) / c + 2);
            if (best < 0 || cost < best) {
                best = cost;
                s = c;
            }
        }
    } else {
        // latency-bound gather: one tile per split where the GPU has room
        // (a wave of at most one CTA per SM); whether the splits of a unit
        // combine in a cluster is decided at launch (attn_cluster_fits)
        const long long nbmax = block == 1 ? d.Ncap : ceil_div(d.Ncap, block);
        rows = (long long)(k_max < nbmax ? k_max : nbmax) * block;
        s = (int)((rows + kTileRows - 1) / kTileRows);
        const int room = kSms / units > 1 ? kSms / units : 1;
        if (s > room) s = room;
        // past 8 splits the partials combine through the workspace (the last CTA
        // of a unit reads them all), which costs more than the extra splits save
        // unless there are too few units to fill the GPU (16-CTA clusters measured
        // no faster than 8: the per-launch chain of dependent loads dominates)
        if (s > kClusterMax && units >= 4) s = kClusterMax;
    }
    const long long smax = (rows + 31) / 32;  // at least 32 positions per split
    if (s > smax) s = (int)smax;
    if (s > kMaxSplits) s = kMaxSplits;
    if (s < 1) s = 1;
    return s;
}

size_t attn_partials_floats(const Dims& d, int splits) {
    return (size_t)d.units() * splits * d.G * kPartStride;
}

static int g_attn_configured[64];

// Clusters of S CTAs need S free SMs in one GPC at once: with ~226 KB of shared
// memory per CTA a B200 holds only 15 clusters of 8 (not 148 / 8), and a 16th
// would wait for a whole wave.  The count comes from the occupancy API, per
// device and kernel configuration, and the cluster combine is used only when
// every unit's cluster is co-resident; otherwise the splits combine through the
// workspace (sized for them in either case).
static int g_max_clusters[64][4][2][2][kClusterMax + 1];  // dev, log2 G, one-tile, contig, S; 0 = unknown

template <int G, int STAGES, bool CONTIG, bool ONE>
static int max_active_clusters(int S) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, 1);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = AttnCfg<G>::smem_bytes(STAGES, true);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_kernel<G, STAGES, true, CONTIG, ONE>, &cfg) != cudaSuccess) {
        cudaGetLastError();  // clear it: the workspace combine is always available
        return -1;
    }
    return n;
}

template <int G>
static bool attn_cluster_fits_g(int dev, bool one_tile, bool contig, int S, int units) {
    const int lg = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
    int& slot = g_max_clusters[dev][lg][one_tile][contig][S];
    if (slot == 0) {
        int n;
        if (!contig) n = one_tile ? max_active_clusters<G, 1, false, true>(S) : max_active_clusters<G, 1, false, false>(S);
        else n = one_tile ? max_active_clusters<G, 1, true, false>(S) : max_active_clusters<G, kRing, true, false>(S);
        slot = n;
    }
    return slot > 0 && units <= slot;
}

static bool attn_cluster_fits(int G, bool one_tile, bool contig, int S, int units) {
    if (S > kClusterMax) return false;
    if (S == 1) return true;  // a cluster of one: no co-scheduling constraint
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    switch (G) {
        case 1: return attn_cluster_fits_g<1>(dev, one_tile, contig, S, units);
        case 2: return attn_cluster_fits_g<2>(dev, one_tile, contig, S, units);
        case 4: return attn_cluster_fits_g<4>(dev, one_tile, contig, S, units);
        case 8: return attn_cluster_fits_g<8>(dev, one_tile, contig, S, units);
        default: return false;
    }
}

struct AttnArgs {
    CUtensorMap kmap, vmap;
    const __nv_bfloat16 *q, *k, *v;
    const int32_t *lens, *idx, *kreq;
    int k_max, block, Hkv, Ncap;
    float sl2;
    int splits;
    float* partials;
    unsigned* counters;
    float* O;
    unsigned* flag;
    int early;
    float* sout;
    float scale;
    float* lse;
};

template <int G, int STAGES, bool CLUSTER, bool CONTIG, bool ONE = false>
static cudaError_t attn_launch_g(dim3 grid, cudaStream_t st, const AttnArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = AttnCfg<G>::smem_bytes(STAGES, CLUSTER);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CLUSTER ? (unsigned)a.splits : 1u;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attn_kernel<G, STAGES, CLUSTER, CONTIG, ONE>, a.kmap, a.vmap, a.q, a.k, a.v, a.lens,
                              a.idx, a.kreq, a.k_max, a.block, a.Hkv, a.Ncap, a.sl2, a.splits, a.partials, a.counters,
                              a.O, a.flag, a.early, a.sout, a.scale, a.lse);
}

template <int G, int STAGES, bool CLUSTER, bool CONTIG, bool ONE = false>
static cudaError_t attn_configure_one() {
    const void* f = (const void*)attn_kernel<G, STAGES, CLUSTER, CONTIG, ONE>;
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         AttnCfg<G>::smem_bytes(STAGES, CLUSTER));
    if (e == cudaSuccess && CLUSTER) e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

template <int G>
static cudaError_t attn_configure() {
    cudaError_t e = cudaSuccess;
    // the gather runs one stage; contiguous tiles one or kRing
    if (e == cudaSuccess) e = attn_configure_one<G, 1, true, false>();
    if (e == cudaSuccess) e = attn_configure_one<G, 1, false, false>();
    if (e == cudaSuccess) e = attn_configure_one<G, 1, true, false, true>();
    if (e == cudaSuccess) e = attn_configure_one<G, 1, false, false, true>();
    if (e == cudaSuccess) e = attn_configure_one<G, 1, true, true>();
    if (e == cudaSuccess) e = attn_configure_one<G, kRing, true, true>();
    if (e == cudaSuccess) e = attn_configure_one<G, 1, false, true>();
    if (e == cudaSuccess) e = attn_configure_one<G, kRing, false, true>();
    return e;
}

template <int G, bool CONTIG>
static cudaError_t attn_dispatch2(bool one_tile, bool cluster, dim3 grid, cudaStream_t st, const AttnArgs& a) {
    if constexpr (!CONTIG) {  // the gather: one stage; one tile a CTA -> the cp.async instance
        if (one_tile)
            return cluster ? attn_launch_g<G, 1, true, false, true>(grid, st, a)
                           : attn_launch_g<G, 1, false, false, true>(grid, st, a);
        return cluster ? attn_launch_g<G, 1, true, false>(grid, st, a) : attn_launch_g<G, 1, false, false>(grid, st, a);
    } else {
        if (cluster)
            return one_tile ? attn_launch_g<G, 1, true, true>(grid, st, a) : attn_launch_g<G, kRing, true, true>(grid, st, a);
        return one_tile ? attn_launch_g<G, 1, false, true>(grid, st, a) : attn_launch_g<G, kRing, false, true>(grid, st, a);
    }
}

template <int G>
static cudaError_t attn_dispatch(bool contig, bool one_tile, bool cluster, dim3 grid, cudaStream_t st,
                                 const AttnArgs& a) {
    return contig ? attn_dispatch2<G, true>(one_tile, cluster, grid, st, a)
                  : attn_dispatch2<G, false>(one_tile, cluster, grid, st, a);
}

// tensor map over a [units * Ncap rows] x [128 dims] bf16 cache, box 64 dims x 128 rows, 128-byte swizzle
static cudaError_t make_row_map(CUtensorMap* map, const void* base, const Dims& d) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)d.units() * (cuuint64_t)d.Ncap};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTileRows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_attn(const void* Q, const void* K, const void* V, const int32_t* lens,
                        const int32_t* idx, const int32_t* kreq, int k_max, int block,
                        const Dims& d, float scale, int splits, float* partials,
                        unsigned* counters, float* O, unsigned* flag, cudaStream_t st, bool early,
                        float* scores_out, bool host_kv, float* lse_out) {
    if (d.units() == 0) return cudaSuccess;
    // scores come with full attention on the tensor-map path only
    if (scores_out && (idx != nullptr || host_kv)) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !g_attn_configured[dev]) {
        if ((e = attn_configure<1>()) != cudaSuccess) return e;
        if ((e = attn_configure<2>()) != cudaSuccess) return e;
        if ((e = attn_configure<4>()) != cudaSuccess) return e;
        if ((e = attn_configure<8>()) != cudaSuccess) return e;
        g_attn_configured[dev] = 1;
    }
    // positions per split (an upper bound): one tile -> single-stage kernel
    long long rows;
    if (idx == nullptr) {
        rows = d.Ncap;
    } else {
        const long long nbmax = block == 1 ? d.Ncap : ceil_div(d.Ncap, block);
        rows = (long long)(k_max < nbmax ? k_max : nbmax) * block;
    }
    // whole 128-row tiles of consecutive cache rows: full attention, or 128-token
    // blocks.  K and V in host memory (index-guided offload) always take the
    // gather, which fetches only the rows in the set, with plain vector loads
    // through the device's mapping of the host pages (no tensor map over them).
    const bool contig = !host_kv && (idx == nullptr || block == kTileRows);
    const long long per_split = contig ? ((rows + splits - 1) / splits + kTileRows - 1) / kTileRows * kTileRows
                                       : (rows + splits - 1) / splits;
    // one tile a CTA: the single-stage kernel (contiguous tiles), or the gather's
    // two-CTAs-an-SM instance (its cp.async copies are kept to device memory)
    const bool one_tile = per_split <= kTileRows && !host_kv;
    const bool cluster = attn_cluster_fits(d.G, one_tile, contig, splits, d.units());
    AttnArgs a;
    memset(&a.kmap, 0, sizeof a.kmap);
    memset(&a.vmap, 0, sizeof a.vmap);
    if (contig) {
        if ((e = make_row_map(&a.kmap, K, d)) != cudaSuccess) return e;
        if ((e = make_row_map(&a.vmap, V, d)) != cudaSuccess) return e;
    }
    a.q = static_cast<const __nv_bfloat16*>(Q);
    a.k = static_cast<const __nv_bfloat16*>(K);
    a.v = static_cast<const __nv_bfloat16*>(V);
    a.lens = lens;
    a.idx = idx;
    a.kreq = kreq;
    a.k_max = k_max;
    a.block = block;
    a.Hkv = d.Hkv;
    a.Ncap = d.Ncap;
    a.sl2 = scale * kLog2e;
    a.splits = splits;
    a.partials = partials;
    a.counters = counters;
    a.O = O;
    a.flag = flag;
    a.early = early ? 1 : 0;
    a.sout = scores_out;
    a.scale = scale;
    a.lse = lse_out;
    dim3 grid(splits, d.units());
    switch (d.G) {
        case 1: e = attn_dispatch<1>(contig, one_tile, cluster, grid, st, a); break;
        case 2: e = attn_dispatch<2>(contig, one_tile, cluster, grid, st, a); break;
        case 4: e = attn_dispatch<4>(contig, one_tile, cluster, grid, st, a); break;
        case 8: e = attn_dispatch<8>(contig, one_tile, cluster, grid, st, a); break;
        default: return cudaErrorInvalidValue;
    }
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa
