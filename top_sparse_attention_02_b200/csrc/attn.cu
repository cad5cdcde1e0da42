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
//   - gather (an index list of tokens): each warp fetches its own 16 rows of
//     every tile with cp.async straight into shared memory, into a per-warp
//     ring of up to 3 tiles, so that all of a CTA's tiles (3 at the 128K
//     shape) are in flight at once; with one tile a CTA the ring is one stage
//     and two CTAs fit an SM.  (K and V in mapped host memory are fetched with
//     16-byte vector loads one tile ahead in registers instead.)  Rows are
//     padded to 272 B so the fragment loads below are free of bank conflicts,
//     and no barrier wider than a warp is needed per tile: a warp only ever
//     reads the rows it copied.  (One TMA bulk copy per 256-byte row was the
//     first design: issuing them cost ~13 ns a copy.)
//   - contiguous tiles (full attention, or a 128-token block): four 2-D TMA
//     tensor loads a tile in the 128-byte swizzle into a 3-stage ring, each
//     stage completing on an mbarrier, refilled as soon as it is consumed.
// Each warp then runs, on its
// 16 rows, the two contractions of flash decoding on the tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate), transposed so that the 16
// rows are the M dimension and the g <= 8 query heads of the group the N
// dimension (one n-tile of 8):
//   S^T = K Q^T    (8 k-steps of 16 dims: 8 MMAs; K fragments by ldmatrix,
//                  Q^T fragments held in registers for the whole kernel),
//   online softmax per head on the S^T fragments (fp32, log2 units),
//   O^T += V^T P^T (8 m-tiles of 16 dims, P split as bf16 hi + bf16 lo so
//                  that the weights keep ~16 bits; V^T fragments by
//                  ldmatrix.trans, P^T fragments from the S^T accumulator by
//                  movmatrix.trans).  In the gather with g <= 4 the n-tile's
//                  columns G .. 2G-1 repeat the heads (Q^T column c is head
//                  c mod G) and carry lo while columns 0 .. G-1 carry hi: one
//                  MMA an m-tile (8), the two column sets summed once at the
//                  end.  With g = 8 there is no spare column, and contiguous
//                  tiles (HBM-bound) keep zero columns: two MMAs an m-tile
//                  (the spare-column form made the 128K full layer 1.5 us
//                  slower).
// A warp-tile is a chain of dependent steps (on sm_100a: ~20 cycles an
// mma.sync, ~30 a shuffle, an exp2 or a shared load), so when a CTA's whole
// range is in its cp.async ring, each warp takes all its 16-row groups in one
// pass: their S^T products are independent MMA chains, one pair of row
// reductions serves them all, and the PV products accumulate in turn.
// With the heads as M instead (padded to 16), each 16 rows took twice the
// MMAs and twice the accumulator registers.  tcgen05's smallest M is 64, so
// a GQA group would leave most of every tcgen05 MMA idle.  The 8 warps are merged at the end into
// the CTA's partial (M, L, acc[128]) per head.  When a unit has at most 8
// splits and every unit's cluster can be resident at once, the splits of a unit
// form one thread-block cluster: output slot q (4 dims of one head) belongs
// to CTA q / ceil(32g / S); each CTA sends every owner its slots of the
// partial and its (M, L) per head with st.async, which counts the bytes on the
// owner's mbarrier, so an owner waits for exactly the bytes it needs (no
// cluster-wide barrier, ~0.5 us less than posted stores and one), then
// combines its slots (no scratch).  Otherwise (more splits, or more clusters
// than fit: a B200 holds only 15 clusters of 8 CTAs of ~226 KB) each CTA
// writes its partial to the workspace and the last CTA of the unit to arrive
// (an atomic counter in the workspace, reset by that CTA) combines the
// partials into O.  (Each warp sending its own partial to the owners, with
// no merge inside the CTA, moved 8x the bytes between SMs: slower.)
//
// Programmatic dependent launch: the kernel may start while the kernel before
// it on the stream is still running.  It waits for it (griddepcontrol.wait)
// before the first read of anything that kernel may have written.  How much it
// does before that wait is the `early` level: 0 nothing; 1 the lengths and k's
// (the decode step's own top-k writes only the indices); 2 also the index list
// and the first tiles' K and V rows (the caller has promised that the kernel
// just before does not write them), so that a reuse layer's gather overlaps the
// end of the layer before it.  Q, the workspace and O are touched only after
// the wait.
#include <cstring>
#include <type_traits>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"

namespace tsa {

constexpr int kMaxSplits = 256;
constexpr int kClusterMax = 8;  // splits per unit that combine inside one (portable) cluster
constexpr int kSms = 148;
constexpr int kPartStride = kD + 4;  // M, L, 2 pad, acc[128]: 528 B, 16-byte aligned
constexpr int kAttnThreads = 256;
constexpr int kAccStride = kD + 4;  // floats per (warp, head) row of the merge buffer: 16-byte rows, no bank conflicts
constexpr int kAttnWarps = 8;
constexpr int kTileRows = 128;                         // 16 rows per warp
constexpr int kRowStride = kD * 2 + 16;                // 272 B: padded so 8 rows hit 8 bank groups
constexpr int kStageBytes = kTileRows * kRowStride * 2;  // K and V of one tile: 68 KB
// cp.async gather: one warp's 16 rows of one tile (K rows, then V rows) form a
// slot; slot (t % STAGES) * 8 + warp holds warp `warp`'s rows of tile t, so a
// CTA whose range is n warp-tiles (16 rows each) uses only slots 0 .. n - 1
// (no ring wrap) and its shared memory is sized by n at launch
constexpr int kSlotBytes = 16 * kRowStride * 2;  // 8.5 KB
constexpr int kRing = 3;                               // tiles in flight (the multi-tile kernel)
#ifndef TSA_WAIT_SPINS
constexpr long kWaitSpins = 1L << 22;  // bounded mbarrier wait (then flag, drain and stop)
#else
constexpr long kWaitSpins = TSA_WAIT_SPINS;  // a debug build's short limit
#endif
constexpr long kRecvSpins = 1L << 22;  // bounded wait for the cluster peers' partials
#ifdef TSA_DEBUG_KNOBS
// Debug build only (never in the product library): the contiguous tile (of CTA
// (0, 0)) whose loads are left out, so that the wait on it runs out; -1: none.
__device__ int g_debug_attn_skip_tile = -1;
#endif

template <int G>
struct AttnCfg {
    // receive area of a cluster of S CTAs: from each source CTA, its partial's
    // float4 slots that this CTA owns (ceil(32G / S) at most: 4 dims of one
    // head a slot), then its (M, L) per head
    __host__ __device__ static constexpr int recv_bytes(int S) {
        return S <= 1 ? 0 : S * ((G * 32 + S - 1) / S) * 16 + S * G * 8;
    }
    static constexpr int recv_max() {
        int m = 0;
        for (int S = 2; S <= kClusterMax; ++S) m = recv_bytes(S) > m ? recv_bytes(S) : m;
        return m;
    }
    static constexpr int kAccBytes = kAttnWarps * G * kAccStride * 4;
    static constexpr int work_bytes(int stages) {
        return stages * kStageBytes > kAccBytes ? stages * kStageBytes : kAccBytes;
    }
    static constexpr int smem_bytes(int stages, bool cluster) {
        return 1024 /* alignment slack */ + work_bytes(stages) + (cluster ? recv_max() : 0);
    }
    // the cp.async gather with `slots` warp-tile slots in use
    static constexpr int slot_work_bytes(int slots) {
        return slots * kSlotBytes > kAccBytes ? slots * kSlotBytes : kAccBytes;
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
// raising the timeout flag, and returns false (the CTA then stops its tile loop;
// see the contiguous-tile loop).  flag == nullptr: no flag (a drain wait).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, unsigned* flag, long spins = kWaitSpins) {
    const unsigned a = smem_u32(bar);
    for (long i = 0; i < spins; ++i) {
        unsigned done;
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
                     : "=r"(done) : "r"(a), "r"(parity) : "memory");
        if (done) return true;
    }
    if (flag) atomicOr(flag, kFlagTimeout);
    return false;
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void st_async_f2(unsigned dst, float x, float y, unsigned bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];\n"
                 ::"r"(dst), "f"(x), "f"(y), "r"(bar) : "memory");
}
// the address of the same shared-memory location in cluster CTA `rank`
__device__ __forceinline__ unsigned cluster_addr(unsigned local, unsigned rank) {
    unsigned r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
// 16 bytes into another cluster CTA's shared memory, counted on that CTA's
// mbarrier (complete_tx): its wait ends once every byte it expects has landed
__device__ __forceinline__ void st_async_f4(unsigned dst, float x, float y, float z, float w, unsigned bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];\n"
                 ::"r"(dst), "f"(x), "f"(y), "f"(z), "f"(w), "r"(bar) : "memory");
}
__device__ __forceinline__ void ldsm_x4(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate (A row-major 16x16 in
// a0..a3, B column-major 16x8 in b0, b1; the PTX ISA's fragment layouts).
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// transpose of an 8x8 b16 matrix held one row pair per lane (lane/4 = row,
// lane%4 = column pair) into the same layout
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
    return d;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
// byte offset of 16-byte chunk `chunk` of row `row` in a tile of padded rows
__device__ __forceinline__ int roff(int row, int chunk) { return row * kRowStride + (chunk << 4); }

// The two contractions of flash decoding on one warp's rows, R groups of 16
// (group q: K at kt[q], V at vt[q], each seen as rows r0 .. r0 + 15 of a tile;
// bit x of vm[q]: row r0 + x of the group is in the set), with one online-
// softmax step over all of them.  The groups' S^T products are independent
// MMA chains and share one pair of row reductions, and the PV products of all
// groups accumulate in turn, so R groups cost far less than R calls of one.
// su_out (CONTIG, R = 1: full attention that also emits its top-k): the scores
// of the group's rows -- scale x the max over the group's heads of q.k, the
// criterion a SELECT layer scores by -- written as S is formed (row first +
// r0 + x), with their top-digit histogram in s_hist.
template <int G, int R, bool CONTIG, bool SPARE>
__device__ __forceinline__ void warp_rows(const unsigned (&kt)[R], const unsigned (&vt)[R], const uint32_t (&vm)[R],
                                          const uint32_t (&qa)[8][2], float (&o)[8][4], float (&m_run)[2],
                                          float (&l_run)[2], float scale_log2, int lane, int r0, float* su_out,
                                          int first, float scale, uint32_t* s_hist) {
    const int g = lane >> 2, t4 = lane & 3;
    // byte offset of 16-byte chunk c of tile row r (padded rows, or the
    // 128-byte swizzle of the TMA tensor loads: two 64-dim halves)
    auto off = [&](int r, int c) -> unsigned {
        if constexpr (CONTIG)
            return (unsigned)((c >> 3) * 64 * kTileRows * 2 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
        else
            return (unsigned)roff(r, c);
    };
    // ---- S^T = K Q^T over each group's 16 rows (M = rows, N = heads)
    // c[q][0], [1]: row g, heads 2t4, 2t4 + 1; [2], [3]: row g + 8
    float c[R][4];
    {
        float sc[R][2][4];  // even / odd k-steps: two chains a group
#pragma unroll
        for (int q = 0; q < R; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[q][0][e] = sc[q][1][e] = 0.f;
        const int m = lane >> 3, i = lane & 7;  // ldmatrix: matrix m, row i
        const int row = r0 + (m & 1) * 8 + i;    // rows +8 (m&1), dims +8 (m>>1)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int q = 0; q < R; ++q) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(kt[q] + off(row, 2 * ks + (m >> 1)), a0, a1, a2, a3);
                mma_bf16(sc[q][ks & 1], a0, a1, a2, a3, qa[ks][0], qa[ks][1]);
            }
#pragma unroll
        for (int q = 0; q < R; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) c[q][e] = sc[q][0][e] + sc[q][1][e];
    }
    const int h0 = 2 * t4, h1 = 2 * t4 + 1;  // this lane's two heads (columns)
    if constexpr (CONTIG && R == 1) {
        const bool va = (vm[0] >> g) & 1u, vb = (vm[0] >> (g + 8)) & 1u;
        if (su_out) {  // uniform: each row's max over the heads < G, across the 4 lanes of the row
            float ea = fmaxf(h0 < G ? c[0][0] : -INFINITY, h1 < G ? c[0][1] : -INFINITY);
            float eb = fmaxf(h0 < G ? c[0][2] : -INFINITY, h1 < G ? c[0][3] : -INFINITY);
#pragma unroll
            for (int o2 = 1; o2 < 4; o2 <<= 1) {
                ea = fmaxf(ea, __shfl_xor_sync(0xffffffffu, ea, o2));
                eb = fmaxf(eb, __shfl_xor_sync(0xffffffffu, eb, o2));
            }
            if (t4 == 0) {  // scale > 0: scale x max = max of the scaled logits
                if (va) {
                    const float v = ea * scale;
                    su_out[first + r0 + g] = v;
                    if (s_hist) atomicAdd(&s_hist[order_key(v) >> 21], 1u);
                }
                if (vb) {
                    const float v = eb * scale;
                    su_out[first + r0 + g + 8] = v;
                    if (s_hist) atomicAdd(&s_hist[order_key(v) >> 21], 1u);
                }
            }
        }
    }
    // ---- online softmax per head (columns of S^T): rows not in the set are -inf
    float z[R][4];
    float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int q = 0; q < R; ++q) {
        const bool va = (vm[q] >> g) & 1u, vb = (vm[q] >> (g + 8)) & 1u;  // rows g, g + 8 in the set
        z[q][0] = va ? c[q][0] * scale_log2 : -INFINITY;
        z[q][1] = va ? c[q][1] * scale_log2 : -INFINITY;
        z[q][2] = vb ? c[q][2] * scale_log2 : -INFINITY;
        z[q][3] = vb ? c[q][3] * scale_log2 : -INFINITY;
        mt[0] = fmaxf(mt[0], fmaxf(z[q][0], z[q][2]));
        mt[1] = fmaxf(mt[1], fmaxf(z[q][1], z[q][3]));
    }
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {  // over the 8 lanes of a t4 (the rows)
        mt[0] = fmaxf(mt[0], __shfl_xor_sync(0xffffffffu, mt[0], o2));
        mt[1] = fmaxf(mt[1], __shfl_xor_sync(0xffffffffu, mt[1], o2));
    }
    float alpha[2], p[R][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float mnew = fmaxf(m_run[j], mt[j]);
        // a head with no finite logit yet keeps m = -inf, alpha = 0 and p = 0
        alpha[j] = m_run[j] == -INFINITY ? 0.f : exp2f(m_run[j] - mnew);
        m_run[j] = mnew;
    }
    float ps[2] = {0.f, 0.f};
#pragma unroll
    for (int q = 0; q < R; ++q) {
#pragma unroll
        for (int e = 0; e < 4; ++e) p[q][e] = z[q][e] == -INFINITY ? 0.f : exp2f(z[q][e] - m_run[e & 1]);
        ps[0] += p[q][0] + p[q][2];
        ps[1] += p[q][1] + p[q][3];
    }
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
        ps[0] += __shfl_xor_sync(0xffffffffu, ps[0], o2);
        ps[1] += __shfl_xor_sync(0xffffffffu, ps[1], o2);
    }
    l_run[0] = l_run[0] * alpha[0] + ps[0];
    l_run[1] = l_run[1] * alpha[1] + ps[1];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[1];
        o[n][2] *= alpha[0];
        o[n][3] *= alpha[1];
    }
    // P^T as the B operand (k = group rows, n = heads), split hi + lo: the
    // accumulator holds row g / heads 2t4.. of each 8x8 block, the operand
    // rows 2t4.. / head g, so each block is transposed in registers
    const int m = lane >> 3, i = lane & 7;  // ldmatrix.trans: matrix m, row i
    const int row = r0 + (m >> 1) * 8 + i;   // rows +8 (m>>1), dims +8 (m&1)
    if constexpr (SPARE) {
        // column c of this lane (2t4 + j) carries part c / G of its head's
        // weight: 0 the bf16 value, 1 the bf16 remainder, 2+ nothing
        auto piece = [&](float v, int part) -> float {
            const float hi = __bfloat162float(__float2bfloat16_rn(v));
            return part == 0 ? hi : (part == 1 ? v - hi : 0.f);
        };
        const int part0 = h0 / G, part1 = h1 / G;
        uint32_t b0[R], b1[R];
#pragma unroll
        for (int q = 0; q < R; ++q) {
            b0[q] = movmatrix_t(pack_bf16(piece(p[q][0], part0), piece(p[q][1], part1)));
            b1[q] = movmatrix_t(pack_bf16(piece(p[q][2], part0), piece(p[q][3], part1)));
        }
        // ---- O^T += V^T P^T over 8 m-tiles of 16 dims, one MMA a group
#pragma unroll
        for (int mt2 = 0; mt2 < 8; ++mt2)
#pragma unroll
            for (int q = 0; q < R; ++q) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(vt[q] + off(row, 2 * mt2 + (m & 1)), a0, a1, a2, a3);
                mma_bf16(o[mt2], a0, a1, a2, a3, b0[q], b1[q]);
            }
    } else {
        uint32_t bh0[R], bh1[R], bl0[R], bl1[R];
#pragma unroll
        for (int q = 0; q < R; ++q) {
            const uint32_t pa = pack_bf16(p[q][0], p[q][1]), pb = pack_bf16(p[q][2], p[q][3]);
            const __nv_bfloat162 ha = *reinterpret_cast<const __nv_bfloat162*>(&pa);
            const __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162*>(&pb);
            const uint32_t la = pack_bf16(p[q][0] - __low2float(ha), p[q][1] - __high2float(ha));
            const uint32_t lb = pack_bf16(p[q][2] - __low2float(hb), p[q][3] - __high2float(hb));
            bh0[q] = movmatrix_t(pa);
            bh1[q] = movmatrix_t(pb);
            bl0[q] = movmatrix_t(la);
            bl1[q] = movmatrix_t(lb);
        }
        // ---- O^T += V^T P^T over 8 m-tiles of 16 dims, hi then lo a group
#pragma unroll
        for (int mt2 = 0; mt2 < 8; ++mt2)
#pragma unroll
            for (int q = 0; q < R; ++q) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(vt[q] + off(row, 2 * mt2 + (m & 1)), a0, a1, a2, a3);
                mma_bf16(o[mt2], a0, a1, a2, a3, bh0[q], bh1[q]);
                mma_bf16(o[mt2], a0, a1, a2, a3, bl0[q], bl1[q]);
            }
    }
}

// CONTIG: every tile is 128 consecutive cache rows (a full-attention range, or
// one 128-token block in block mode) and arrives by 2-D TMA tensor loads in the
// 128-byte-swizzled layout (4 loads per tile) into a ring of STAGES tiles;
// otherwise (a gather) rows are padded to 272 bytes.
// ASYNC (gather only): rows are copied straight into shared memory (cp.async)
// into per-warp slots, a ring of STAGES tiles; launched two CTAs an SM when the
// slots a CTA uses allow it.  Otherwise (K and V in mapped host memory) each
// warp loads its rows into registers one tile ahead and stores them.
template <int G, int STAGES, bool CLUSTER, bool CONTIG, bool ASYNC>
__global__ void __launch_bounds__(kAttnThreads, ASYNC ? 2 : 1)
attn_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
            const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
            const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ lens,
            const int32_t* __restrict__ idx, const int32_t* __restrict__ kreq, int k_max,
            int block, int Hkv, int Ncap, float scale_log2, int S, float* __restrict__ part,
            unsigned* __restrict__ counters, float* __restrict__ O, unsigned* __restrict__ flag, int early,
            float* __restrict__ sout, float scale, float* __restrict__ lse, int work,
            uint32_t* __restrict__ hout) {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "the group's heads fill a power-of-two part of one n-tile");
    using Cfg = AttnCfg<G>;
    // the gather (latency-bound: its MMAs are on the chain) puts P's low part
    // in the n-tile's spare columns; contiguous tiles (HBM-bound, the math
    // hidden under the stream) keep zero columns and a second MMA, which
    // measured faster there (128K full layer 86.1 against 88.0 us cold)
    constexpr bool SPARE = G <= 4 && !CONTIG;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // 1024-byte aligned work area (the swizzled layout needs it)
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ float s_wm[kAttnWarps][G], s_wl[kAttnWarps][G];
    __shared__ int s_last;
    __shared__ int s_fail;  // CONTIG: a bounded wait gave up; the CTA stops its tile loop
    __shared__ __align__(8) uint64_t s_bar[STAGES];
    __shared__ int s_first[STAGES];  // CONTIG: first cache row of the tile in each stage, or -1
    __shared__ __align__(8) uint64_t s_rbar;  // cluster combine: the peers' slices have landed

    const int s = blockIdx.x, unit = blockIdx.y;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;  // mma fragment coordinates
    // early >= 1: the kernel before this one did not write the lengths or the
    // k's (the decode step's own top-k), so they are read before waiting on it;
    // early == 2: neither the index list nor K and V (the caller's promise), so
    // the first tiles are fetched before the wait too (below)
    int len = 0, kreq_b = k_max;
    if (early) {
        len = __ldcg(lens + b);
        if (kreq) kreq_b = __ldcg(kreq + b);
    }
    // Q's lines into L2 while the previous kernel finishes (G x 256 bytes)
    if (tid < 2 * G) prefetch_l2(Q + (size_t)unit * G * kD + tid * 64);
    // The set-up below reads nothing the previous kernel writes, so it runs
    // before the wait on it: out of the chain after the wait (barrier inits and
    // their fence, a CTA barrier, the cluster arrive).
    // Full attention handing on its top-k: a histogram of the emitted scores'
    // top 11 key bits (the top-k's first radix digit), past the work area.
    uint32_t* const s_hist = (CONTIG && sout && hout)
        ? reinterpret_cast<uint32_t*>(smem + work + (CLUSTER ? Cfg::recv_bytes(S) : 0)) : nullptr;
    const bool ccomb = CLUSTER && S > 1;  // the splits combine in this cluster (uniform)
    if (s_hist)
        for (int i = tid; i < kHistBins; i += kAttnThreads) s_hist[i] = 0u;
    if (tid == 0) {
        s_fail = 0;
#pragma unroll
        for (int i = 0; i < STAGES; ++i) mbar_init(&s_bar[i], CONTIG ? 1 : kTileRows);
        if (ccomb) {
            // every CTA of the cluster sends this CTA the slots of its partial
            // that this CTA owns, and its (M, L) per head
            const int per = ceil_div(G * 32, S);
            const int own = max(0, min(per, G * 32 - s * per));
            mbar_init(&s_rbar, 1);
            mbar_arrive_expect_tx(&s_rbar, (unsigned)(S * (own * 16 + G * 8)));
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    // every CTA of the cluster has started and armed its receive barrier once
    // this phase completes (waited for just before the first remote store)
    if (ccomb) asm volatile("barrier.cluster.arrive.relaxed;\n" ::: "memory");
    if (early < 2) {
        griddep_wait();
        griddep_launch();
    }
    // Gather: the index entries of this lane's rows (lanes 0-15: rows r0 +
    // lane) in the first ring stages, loaded at once for the range this split
    // has when every unit attends to k_max entries -- before the lengths and
    // k's have arrived.  Checked against the real range below (the same range
    // unless k_b < k_max), and loaded again where it differs.
    constexpr int NEV = CONTIG ? 1 : (ASYNC ? STAGES : 1);
    const int32_t* iu = idx ? idx + (size_t)unit * k_max : nullptr;
    const int r0 = warp * 16;  // this warp's rows in a tile
    int ev[NEV];
    int spec_p0 = -1;
    if constexpr (!CONTIG) {
        if (iu != nullptr) {
            const int npos_s = k_max * block;
            const int chunk_s = ceil_div(npos_s, S);
            spec_p0 = min(s * chunk_s, npos_s);
            const int spec_p1 = min(spec_p0 + chunk_s, npos_s);
#pragma unroll
            for (int i = 0; i < NEV; ++i) {
                const int pos = spec_p0 + i * kTileRows + r0 + lane;
                ev[i] = (lane < 16 && pos < spec_p1) ? __ldcg(iu + (block == 1 ? pos : pos / block)) : -1;
            }
        }
    }
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
    const __nv_bfloat16* Ku = K + (size_t)unit * Ncap * kD;
    const __nv_bfloat16* Vu = V + (size_t)unit * Ncap * kD;

    // cache row of position pos given its index entry e (token mode: the row;
    // block mode: the block), or -1 (skipped entry, tail of a partial block)
    auto row_check = [&](int pos, int e) -> int {
        if (block == 1) {
            if (e >= len) {
                atomicOr(flag, kFlagBounds);
                return -1;
            }
            return e < 0 ? -1 : e;
        }
        const int slot = pos / block;
        if (e >= nb) {
            atomicOr(flag, kFlagBounds);
            return -1;
        }
        if (e < 0) return -1;
        const int r = e * block + (pos - slot * block);
        return r < len ? r : -1;
    };
    auto row_of = [&](int pos) -> int {
        if (iu == nullptr) return pos;
        return row_check(pos, __ldcg(iu + (block == 1 ? pos : pos / block)));
    };
    // CONTIG: the tile's first cache row (dense: its position; block mode: the
    // chosen block's first row), or -1 when the block entry is absent
    auto tile_first = [&](int t) -> int {
        const int pos0 = p0 + t * kTileRows;
        if (t >= ntiles) return -1;
        if (iu == nullptr) return pos0;
        const int e = __ldcg(iu + pos0 / kTileRows);
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
#ifdef TSA_DEBUG_KNOBS
        if (t == g_debug_attn_skip_tile && blockIdx.x == 0 && blockIdx.y == 0) return;  // neither armed nor loaded
#endif
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
    // CONTIG: the first STAGES tiles' block indices in one round, then their loads
    int next_first = -1;  // CONTIG, thread 0: first row of the tile that refills the stage next
    int issued = 0;       // CONTIG, thread 0: tiles whose loads have been issued
    if constexpr (CONTIG) {
        if (tid == 0) {
            issued = min(ntiles, STAGES);
            int f[STAGES];
#pragma unroll
            for (int t = 0; t < STAGES; ++t) f[t] = tile_first(t);
#pragma unroll
            for (int t = 0; t < STAGES; ++t) stage_contig(t, f[t]);
        }
    }

    // Gather: each warp copies its own 16 rows of a tile (a half-warp per
    // 256-byte row; lane l takes 16-byte chunk l & 15 of rows (l >> 4), +2,
    // ..., +14) into its rows of the padded tile, and only that warp reads
    // them: no TMA queue (one 256-byte bulk copy per row issued at ~13 ns a
    // copy per SM, which bounded short gathers) and no CTA barrier per tile.
    // Rows not in the set are zeros (their weight is 0, and 0 x NaN = NaN).
    const int hl = lane >> 4, c16 = lane & 15;
    // this lane's cache row of tile t (lanes 0-15: rows r0 + lane), or -1
    auto my_row = [&](int t) -> int {
        int myrow = -1;
        if (lane < 16) {
            const int pos = p0 + t * kTileRows + r0 + lane;
            if (pos < p1) myrow = row_of(pos);
        }
        return myrow;
    };
    // the rows of the first NEV tiles: their index entries all in flight at
    // once (the speculative loads above where the range agrees)
    int rows0[NEV];
    if constexpr (!CONTIG) {
        const bool spec = iu != nullptr && p0 == spec_p0;
        int e[NEV];
#pragma unroll
        for (int i = 0; i < NEV; ++i) {
            const int pos = p0 + i * kTileRows + r0 + lane;
            e[i] = -1;
            if (iu != nullptr && lane < 16 && pos < p1) e[i] = spec ? ev[i] : __ldcg(iu + (block == 1 ? pos : pos / block));
        }
#pragma unroll
        for (int i = 0; i < NEV; ++i) {
            const int pos = p0 + i * kTileRows + r0 + lane;
            rows0[i] = -1;
            if (lane < 16 && pos < p1) rows0[i] = iu != nullptr ? row_check(pos, e[i]) : pos;
        }
    }
    // register path (K and V in host memory): tile t's rows into registers
    uint4 pk[ASYNC ? 1 : 8], pv[ASYNC ? 1 : 8];
    uint32_t vm_next = 0;
    auto fetch = [&](int t, int myrow) {
        if constexpr (!CONTIG && !ASYNC) {
            vm_next = __ballot_sync(0xffffffffu, myrow >= 0) & 0xffffu;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int rr = __shfl_sync(0xffffffffu, myrow, hl + 2 * j);
                pk[j] = rr >= 0 ? ld_stream(Ku + (size_t)rr * kD + 8 * c16) : make_uint4(0, 0, 0, 0);
                pv[j] = rr >= 0 ? ld_stream(Vu + (size_t)rr * kD + 8 * c16) : make_uint4(0, 0, 0, 0);
            }
        }
    };
    // cp.async path: tile t's rows of this warp (this lane's: myrow) into its
    // slot of ring stage st (not committed here); returns the tile's row mask.
    // A warp with no position of the CTA's range in tile t writes nothing (its
    // slot may lie past the shared memory a short range is given).
    auto issue_async = [&](int t, int st, int myrow) -> uint32_t {
        if (p0 + t * kTileRows + r0 >= p1) return 0u;  // warp-uniform
        const uint32_t vm = __ballot_sync(0xffffffffu, myrow >= 0) & 0xffffu;
        unsigned char* kw = smem + (st * kAttnWarps + warp) * kSlotBytes;
        unsigned char* vw = kw + 16 * kRowStride;
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
        return vm;
    };
    // masks of the tiles in the ring, oldest first (a shift register, so it
    // stays in registers)
    uint32_t vmr[ASYNC ? STAGES : 1];
#pragma unroll
    for (int i = 0; i < (ASYNC ? STAGES : 1); ++i) vmr[i] = 0u;
    if constexpr (!CONTIG) {
        if constexpr (ASYNC) {  // the whole ring in flight (empty groups past the last tile)
#pragma unroll
            for (int i = 0; i < STAGES; ++i) {
                if (i < ntiles) vmr[i] = issue_async(i, i, rows0[i < NEV ? i : 0]);
                asm volatile("cp.async.commit_group;\n" ::: "memory");
            }
        } else if (ntiles > 0) {
            fetch(0, rows0[0]);
        }
    }
    if (early >= 2) {  // everything above read only what the caller promised is not being written
        griddep_wait();
        griddep_launch();
    }

    // B fragments of Q^T (bf16, unscaled: the scale is applied to S in fp32):
    // column g = query head g mod G of the group, rows = dims.  (G <= 4: the
    // columns past G repeat the heads, so every lane's softmax state is that
    // of real heads and the P^T columns past G can carry P's low parts.)
    uint32_t qa[8][2];
    {
        const bool live = SPARE || g < G;  // without spare columns, columns past G are zero
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(Q + ((size_t)unit * G + (g & (G - 1))) * kD);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qa[ks][0] = live ? qrow[ks * 8 + t4] : 0u;       // dims 16ks + 2t4, +1
            qa[ks][1] = live ? qrow[ks * 8 + 4 + t4] : 0u;   // dims 16ks + 8 + 2t4, +1
        }
    }
    // O^T fragments: o[mt][0], [1] = dim 16mt + g, heads 2t4, 2t4 + 1; [2], [3] = dim 16mt + g + 8
    float o[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
    // this warp's running max / sum for heads 2t4 and 2t4 + 1 (equal across the lanes of a t4)
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

    const unsigned sbase = smem_u32(smem);
    // this warp's 16 rows of one tile (K at kt, V at vt; bit i of vm: row r0 + i
    // is in the set); sout: the emitted scores (full attention handing on its top-k)
    float* const su_out = (CONTIG && sout) ? sout + (size_t)unit * Ncap : nullptr;
    auto warp_tile = [&](unsigned kt, unsigned vt, uint32_t vm, int first) {
        const unsigned kk[1] = {kt}, vv[1] = {vt};
        const uint32_t mm[1] = {vm};
        warp_rows<G, 1, CONTIG, SPARE>(kk, vv, mm, qa, o, m_run, l_run, scale_log2, lane, r0, su_out, first, scale,
                                       s_hist);
    };

    if constexpr (CONTIG) {
        int t = 0;
        for (; t < ntiles; ++t) {
            if (tid == 0) next_first = tile_first(t + STAGES);  // in flight during this tile
            // tile t has landed (on a timeout: flag, and the whole CTA stops below)
            if (!mbar_wait(&s_bar[t % STAGES], (unsigned)(t / STAGES) & 1u, flag)) s_fail = 1;
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
            // s_fail is written only before the barrier above and read only
            // between it and the one below, so every thread sees the same value
            if (s_fail) break;
            const int nv = tile_rows - r0;
            const uint32_t vm = nv >= 16 ? 0xffffu : (nv > 0 ? (1u << nv) - 1u : 0u);
            if (vm) {  // warp-uniform
                const unsigned kt = sbase + st * kStageBytes;
                warp_tile(kt, kt + 2 * 64 * kTileRows * 2, vm, first);
            }
            __syncthreads();  // every warp is done with this stage
            if (tid == 0 && t + STAGES < ntiles) {  // refill it (nothing past the end)
                stage_contig(t + STAGES, next_first);
                ++issued;
            }
        }
        // after a timeout: wait (bounded, no second flag) for the loads still in
        // flight, so that none lands in this SM's shared memory after the CTA
        // has gone; the output is then unspecified, and the flag says so
        if (t < ntiles && tid == 0)
            for (int j = t; j < issued; ++j) mbar_wait(&s_bar[j % STAGES], (unsigned)(j / STAGES) & 1u, nullptr);
    } else if constexpr (ASYNC) {
        if (ntiles <= STAGES) {
            // the whole range is in the ring: once it has landed, every row
            // group of this warp in one pass (groups past the last non-empty
            // one skipped; masks are warp-uniform)
            asm volatile("cp.async.wait_all;\n" ::: "memory");
            __syncwarp();
            int nw = 0;
#pragma unroll
            for (int q = 0; q < STAGES; ++q)
                if (vmr[q]) nw = q + 1;
            auto groups = [&](auto rc) {
                constexpr int R = decltype(rc)::value;
                unsigned kk[R], vv[R];
                uint32_t mm[R];
#pragma unroll
                for (int q = 0; q < R; ++q) {
                    kk[q] = sbase + (unsigned)((q * kAttnWarps + warp) * kSlotBytes) - (unsigned)(r0 * kRowStride);
                    vv[q] = kk[q] + 16 * kRowStride;
                    mm[q] = vmr[q];
                }
                warp_rows<G, R, false, SPARE>(kk, vv, mm, qa, o, m_run, l_run, scale_log2, lane, r0, nullptr, 0,
                                              scale, nullptr);
            };
            if constexpr (STAGES >= 3) {
                if (nw == 3) groups(std::integral_constant<int, 3>{});
            }
            if constexpr (STAGES >= 2) {
                if (nw == 2) groups(std::integral_constant<int, 2>{});
            }
            if (nw == 1) groups(std::integral_constant<int, 1>{});
            static_assert(STAGES <= 3, "the one-pass branch covers rings of up to 3 tiles");
        } else {  // a longer range streams through the ring, a tile at a time
            for (int t = 0; t < ntiles; ++t) {
                // this lane's copies of tile t have landed (at most STAGES - 1 newer
                // groups still pending), then the warp's
                asm volatile("cp.async.wait_group %0;\n" ::"n"(STAGES - 1) : "memory");
                __syncwarp();
                const int st = t % STAGES;
                // the slot's rows seen as rows r0 .. r0 + 15 of a tile (the math's row offsets)
                const unsigned ks = sbase + (unsigned)((st * kAttnWarps + warp) * kSlotBytes) - (unsigned)(r0 * kRowStride);
                if (vmr[0]) warp_tile(ks, ks + 16 * kRowStride, vmr[0], 0);
                __syncwarp();  // the math has read these rows before the stage is refilled
#pragma unroll
                for (int i = 0; i + 1 < STAGES; ++i) vmr[i] = vmr[i + 1];
                vmr[STAGES - 1] = t + STAGES < ntiles ? issue_async(t + STAGES, st, my_row(t + STAGES)) : 0u;
                asm volatile("cp.async.commit_group;\n" ::: "memory");
            }
        }
        asm volatile("cp.async.wait_all;\n" ::: "memory");  // nothing in flight over the merge below
    } else {
        unsigned char* kw = smem + r0 * kRowStride;
        unsigned char* vw = smem + (kTileRows + r0) * kRowStride;
        for (int t = 0; t < ntiles; ++t) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                *reinterpret_cast<uint4*>(kw + (hl + 2 * j) * kRowStride + 16 * c16) = pk[j];
                *reinterpret_cast<uint4*>(vw + (hl + 2 * j) * kRowStride + 16 * c16) = pv[j];
            }
            const uint32_t vm = vm_next;
            __syncwarp();
            if (t + 1 < ntiles) fetch(t + 1, my_row(t + 1));  // the next tile's loads fly during this tile's math
            if (vm) warp_tile(sbase, sbase + kTileRows * kRowStride, vm, 0);
            __syncwarp();  // the math has read these rows before the next store
        }
    }
    // spare columns: head h's output is the sum of columns h (hi) and h + G (lo)
    if constexpr (SPARE && (G == 4 || G == 2)) {
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[n][e] += __shfl_xor_sync(0xffffffffu, o[n][e], G / 2);
    } else if constexpr (SPARE && G == 1) {
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            o[n][0] += o[n][1];
            o[n][2] += o[n][3];
        }
    }
    __syncthreads();

    // ---- merge the 8 warps: each warp's (m, l, o) for heads < G
    float* s_acc = reinterpret_cast<float*>(smem);  // [kAttnWarps][G][kAccStride], over the staging ring
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int h = 2 * t4 + j;
        if (h < G) {
            float* row = s_acc + (warp * G + h) * kAccStride;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                row[16 * n + g] = o[n][j];
                row[16 * n + g + 8] = o[n][j + 2];
            }
            if (g == 0) {
                s_wm[warp][h] = m_run[j];
                s_wl[warp][h] = l_run[j];
            }
        }
    }
    __syncthreads();
    if (s_hist) {  // this CTA's counts into the unit's histogram (read once this grid is done)
        uint32_t* hu = hout + (size_t)unit * kHistBins;
        for (int i = tid; i < kHistBins; i += kAttnThreads)
            if (const uint32_t c = s_hist[i]) atomicAdd(&hu[i], c);
    }
    const int nslots = G * 32;  // (head, quad of dims) output slots: thread tid owns slot tid
    const bool has_slot = tid < nslots;
    const int h_me = tid >> 5, qd_me = tid & 31;
    // the CTA's (M, L, acc) for head h_me: every slot thread of the head forms
    // M and L itself from the 8 warps' (m, l) (no extra barrier)
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    float M_me = -INFINITY, L_me = 0.f;
    if (has_slot) {
        float wm[kAttnWarps];
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            wm[w] = s_wm[w][h_me];
            M_me = fmaxf(M_me, wm[w]);
        }
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            const float sc = (wm[w] == -INFINITY || M_me == -INFINITY) ? 0.f : exp2f(wm[w] - M_me);
            L_me += s_wl[w][h_me] * sc;
            const float4 a = *reinterpret_cast<const float4*>(s_acc + (w * G + h_me) * kAccStride + 4 * qd_me);
            A.x += a.x * sc;
            A.y += a.y * sc;
            A.z += a.z * sc;
            A.w += a.w * sc;
        }
    }

    if constexpr (CLUSTER) {
        if (S == 1) {  // nothing to combine
            if (has_slot) {
                const float L = L_me;
                float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
                if (L > 0.f) {
                    const float inv = __fdividef(1.f, L);  // ~2 ulp, ~3x cheaper than IEEE 1/L here
                    r = make_float4(A.x * inv, A.y * inv, A.z * inv, A.w * inv);
                }
                *reinterpret_cast<float4*>(O + ((size_t)unit * G + h_me) * kD + 4 * qd_me) = r;
                if (lse && qd_me == 0) lse[(size_t)unit * G + h_me] = L > 0.f ? M_me + log2f(L) : -INFINITY;
            }
            return;
        }
        // the S splits of this unit are the S CTAs of this cluster (rank =
        // split).  Output slot q (4 dims of one head) is owned by CTA q / per;
        // each CTA sends every owner its slots of its merged partial and its
        // (M, L) per head with st.async, counted on the owner's barrier, so an
        // owner waits only for the bytes it needs (no cluster-wide barrier).
        const int per = ceil_div(nslots, S);
        float4* recv = reinterpret_cast<float4*>(smem + work);      // [src][per]
        float2* rml = reinterpret_cast<float2*>(recv + S * per);    // [src][G]: (M, L)
        const unsigned rbar = smem_u32(&s_rbar);
        asm volatile("barrier.cluster.wait;\n" ::: "memory");  // every peer has armed its barrier
        if (has_slot) {
            const int owner = tid / per, lslot = tid - owner * per;
            st_async_f4(cluster_addr(smem_u32(recv + s * per + lslot), owner), A.x, A.y, A.z, A.w,
                        cluster_addr(rbar, owner));
            if (qd_me < S)  // head h_me's (M, L) to CTA qd_me
                st_async_f2(cluster_addr(smem_u32(rml + s * G + h_me), qd_me), M_me, L_me,
                            cluster_addr(rbar, qd_me));
        }
        // this CTA's slices: one bounded wait, the same outcome for the whole CTA
        const bool ok = mbar_wait(&s_rbar, 0u, nullptr, kRecvSpins);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(flag, kFlagTimeout);
            return;  // the output is unspecified, and the flag says so
        }
        // one thread an owned slot, over the S sources
        const int own = min(per, nslots - s * per);
        if (tid < own) {
            const int slot = s * per + tid;
            const int h = slot >> 5, qd = slot & 31;
            // every source's (M, L) and slot first (no branch between the loads)
            float2 ml[kClusterMax];
            float4 ov[kClusterMax];
#pragma unroll
            for (int j = 0; j < kClusterMax; ++j) {
                const bool v = j < S;
                ml[j] = v ? rml[j * G + h] : make_float2(-INFINITY, 0.f);
                ov[j] = v ? recv[j * per + tid] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float M = ml[0].x;
#pragma unroll
            for (int j = 1; j < kClusterMax; ++j) M = fmaxf(M, ml[j].x);
            float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
            float den = 0.f;
#pragma unroll
            for (int j = 0; j < kClusterMax; ++j) {
                const float w = ml[j].x == -INFINITY ? 0.f : exp2f(ml[j].x - M);
                den += w * ml[j].y;
                num.x += w * ov[j].x;
                num.y += w * ov[j].y;
                num.z += w * ov[j].z;
                num.w += w * ov[j].w;
            }
            float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
            if (den > 0.f) {
                const float inv = __fdividef(1.f, den);  // ~2 ulp, ~3x cheaper than IEEE 1/den here
                r = make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
            }
            *reinterpret_cast<float4*>(O + ((size_t)unit * G + h) * kD + 4 * qd) = r;
            if (lse && qd == 0) lse[(size_t)unit * G + h] = den > 0.f ? M + log2f(den) : -INFINITY;
        }
        return;  // nothing of this CTA is read remotely: CTAs may leave in any order
    } else {
        if (has_slot) {
            float* pu = part + (((size_t)unit * S + s) * G + h_me) * kPartStride;
            *reinterpret_cast<float4*>(pu + 4 + 4 * qd_me) = A;
            if (qd_me == 0) *reinterpret_cast<float2*>(pu) = make_float2(M_me, L_me);
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
            if (den > 0.f) {
                const float inv = __fdividef(1.f, den);
                r = make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
            }
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
        if (s > room) {
            // token gathers: two CTAs an SM when a CTA's range fits 12 warp-tiles
            // (192 rows, ~102 KB of staging); more, shorter CTAs shorten the
            // chain of tiles each warp works through
            const int room2 = 2 * kSms / units > 1 ? 2 * kSms / units : 1;
            const int s2 = s < room2 ? s : room2;
            s = (block == 1 && (rows + s2 - 1) / s2 <= 12 * 16) ? s2 : room;
        }
        // past 8 splits the partials combine through the workspace (the last CTA
        // of a unit reads them all), which costs more than the extra splits save
        // unless there are too few units to fill the GPU (16-CTA clusters measured
        // no faster than 8: the per-launch chain of dependent loads dominates)
        // (16-CTA clusters of short ranges, measured at the 128K shape: the
        // CTAs pack two to an SM and the 16-way combine costs more than the
        // shorter ranges save)
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
// Instance of the kernel a launch takes (besides G and the cluster choice):
// contiguous tiles in a 1-stage or kRing-stage TMA ring; or the gather, through
// registers (host memory), or by cp.async in a 1-stage or kRing-stage ring.
enum AttnVariant { kContig1 = 0, kContigRing = 1, kGatherReg = 2, kGatherAsync1 = 3, kGatherAsyncRing = 4, kVariants = 5 };

// co-resident clusters by (device, log2 G, variant, S, warp-tile slots of the
// cp.async gather or 0); 0 = not queried yet
constexpr int kCacheDevs = 16;
static int g_max_clusters[kCacheDevs][4][kVariants][kClusterMax + 1][3 * kAttnWarps + 1][2];

// the work area (staging, merge buffer) of an instance: the cp.async gather by
// the slots its CTAs use, every other instance its whole ring
template <int G, int STAGES, bool CONTIG, bool ASYNC>
static int work_bytes_of(int slots) {
    return (ASYNC && !CONTIG) ? AttnCfg<G>::slot_work_bytes(slots) : AttnCfg<G>::work_bytes(STAGES);
}

// dynamic shared memory of a launch: the work area, the cluster's receive
// area, and the emitted scores' histogram
template <int G, int STAGES, bool CLUSTER, bool CONTIG, bool ASYNC>
static int smem_of(int S, int slots, bool hist) {
    return 1024 + work_bytes_of<G, STAGES, CONTIG, ASYNC>(slots) + (CLUSTER ? AttnCfg<G>::recv_bytes(S) : 0) +
           (hist ? kHistBins * 4 : 0);
}

template <int G, int STAGES, bool CONTIG, bool ASYNC>
static int max_active_clusters(int S, int slots, bool hist) {
    const void* f = (const void*)attn_kernel<G, STAGES, true, CONTIG, ASYNC>;
    const int smem = smem_of<G, STAGES, true, CONTIG, ASYNC>(S, slots, hist);
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, f) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    if (smem > fa.maxDynamicSharedSizeBytes) return -1;  // past what the kernel was configured for: no cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, 1);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_kernel<G, STAGES, true, CONTIG, ASYNC>, &cfg) != cudaSuccess) {
        cudaGetLastError();  // clear it: the workspace combine is always available
        return -1;
    }
    return n;
}

template <int G>
static int max_clusters_g(int var, int S, int slots, bool hist) {
    switch (var) {
        case kContig1: return max_active_clusters<G, 1, true, false>(S, 0, hist);
        case kContigRing: return max_active_clusters<G, kRing, true, false>(S, 0, hist);
        case kGatherReg: return max_active_clusters<G, 1, false, false>(S, 0, hist);
        case kGatherAsync1: return max_active_clusters<G, 1, false, true>(S, slots, hist);
        default: return max_active_clusters<G, kRing, false, true>(S, slots, hist);
    }
}

// whether the S splits of every unit can combine in a cluster: every cluster
// resident at once, with the shared memory the launch needs
static bool attn_cluster_fits(int G, int var, int S, int units, int slots, bool hist) {
    if (S > kClusterMax) return false;
    if (S == 1) return true;  // a cluster of one: no co-scheduling constraint
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    if (var != kGatherAsync1 && var != kGatherAsyncRing) slots = 0;
    auto query = [&]() {
        switch (G) {
            case 1: return max_clusters_g<1>(var, S, slots, hist);
            case 2: return max_clusters_g<2>(var, S, slots, hist);
            case 4: return max_clusters_g<4>(var, S, slots, hist);
            case 8: return max_clusters_g<8>(var, S, slots, hist);
            default: return -1;
        }
    };
    int n;
    if (dev < kCacheDevs) {
        const int lg = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
        int& c = g_max_clusters[dev][lg][var][S][slots][hist ? 1 : 0];
        if (c == 0) c = query();
        n = c;
    } else {
        n = query();
    }
    return n > 0 && units <= n;
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
    int slots;       // the cp.async gather: warp-tile slots its CTAs use
    uint32_t* hout;  // with sout: the units' top-digit histograms of the emitted scores
};

template <int G, int STAGES, bool CLUSTER, bool CONTIG, bool ASYNC = false>
static cudaError_t attn_launch_g(dim3 grid, cudaStream_t st, const AttnArgs& a) {
    const int work = work_bytes_of<G, STAGES, CONTIG, ASYNC>(a.slots);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem_of<G, STAGES, CLUSTER, CONTIG, ASYNC>(a.splits, a.slots, a.sout && a.hout);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CLUSTER ? (unsigned)a.splits : 1u;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attn_kernel<G, STAGES, CLUSTER, CONTIG, ASYNC>, a.kmap, a.vmap, a.q, a.k, a.v, a.lens,
                              a.idx, a.kreq, a.k_max, a.block, a.Hkv, a.Ncap, a.sl2, a.splits, a.partials, a.counters,
                              a.O, a.flag, a.early, a.sout, a.scale, a.lse, work, a.hout);
}

template <int G, int STAGES, bool CLUSTER, bool CONTIG, bool ASYNC = false>
static cudaError_t attn_configure_one() {
    const void* f = (const void*)attn_kernel<G, STAGES, CLUSTER, CONTIG, ASYNC>;
    // contiguous tiles may carry the emitted scores' histogram (8 KB more);
    // at most what the device allows next to the kernel's static shared
    // memory (a cluster launch that would need more combines in the workspace)
    int dev = 0, optin = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, f);
    if (e != cudaSuccess) return e;
    const int want = AttnCfg<G>::smem_bytes(STAGES, CLUSTER) + (CONTIG ? kHistBins * 4 : 0);
    const int cap = optin - (int)fa.sharedSizeBytes;
    e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, want < cap ? want : cap);
    if (e == cudaSuccess && CLUSTER) e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

template <int G>
static cudaError_t attn_configure() {
    cudaError_t e = cudaSuccess;
    // contiguous tiles: one stage or kRing; the gather: registers, or cp.async
    // with one stage or kRing
#define TSA_CONF(ST, CONTIG, ASYNC)                                                      \
    if (e == cudaSuccess) e = attn_configure_one<G, ST, true, CONTIG, ASYNC>();   \
    if (e == cudaSuccess) e = attn_configure_one<G, ST, false, CONTIG, ASYNC>();
    TSA_CONF(1, true, false)
    TSA_CONF(kRing, true, false)
    TSA_CONF(1, false, false)
    TSA_CONF(1, false, true)
    TSA_CONF(kRing, false, true)
#undef TSA_CONF
    return e;
}

template <int G, int STAGES, bool CONTIG, bool ASYNC>
static cudaError_t attn_launch_c(bool cluster, dim3 grid, cudaStream_t st, const AttnArgs& a) {
    return cluster ? attn_launch_g<G, STAGES, true, CONTIG, ASYNC>(grid, st, a)
                   : attn_launch_g<G, STAGES, false, CONTIG, ASYNC>(grid, st, a);
}

template <int G>
static cudaError_t attn_dispatch(int var, bool cluster, dim3 grid, cudaStream_t st, const AttnArgs& a) {
    switch (var) {
        case kContig1: return attn_launch_c<G, 1, true, false>(cluster, grid, st, a);
        case kContigRing: return attn_launch_c<G, kRing, true, false>(cluster, grid, st, a);
        case kGatherReg: return attn_launch_c<G, 1, false, false>(cluster, grid, st, a);
        case kGatherAsync1: return attn_launch_c<G, 1, false, true>(cluster, grid, st, a);
        default: return attn_launch_c<G, kRing, false, true>(cluster, grid, st, a);
    }
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
                        unsigned* counters, float* O, unsigned* flag, cudaStream_t st, int early,
                        float* scores_out, bool host_kv, float* lse_out, uint32_t* hist_out) {
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
    // one tile a CTA: the single-stage kernel (contiguous tiles), or the gather's
    // two-CTAs-an-SM instance; several: the 3-stage rings.  K and V in host
    // memory: the register gather (cp.async is kept to device memory)
    auto per_split_of = [&](int S) {
        return contig ? ((rows + S - 1) / S + kTileRows - 1) / kTileRows * kTileRows : (rows + S - 1) / S;
    };
    auto variant_of = [&](int S) {
        const bool one_tile = per_split_of(S) <= kTileRows;
        return contig ? (one_tile ? kContig1 : kContigRing)
                      : host_kv ? kGatherReg : one_tile ? kGatherAsync1 : kGatherAsyncRing;
    };
    // warp-tile slots of the cp.async gather: its range's 16-row groups, at
    // most the ring's
    auto slots_of = [&](int S, int var) {
        const long long wt = (per_split_of(S) + 15) / 16;
        const int cap = var == kGatherAsync1 ? kAttnWarps : kRing * kAttnWarps;
        return (int)(wt < cap ? (wt < 1 ? 1 : wt) : cap);
    };
    // Early inputs (the caller's promise): this launch's gathers are meant to
    // run while the launch before it on the stream finishes, so its clusters
    // must find room beside that launch's.  When 2 x units clusters of
    // `splits` CTAs cannot be resident at once (a B200 holds 15 clusters of 8
    // one-CTA-an-SM gathers, 22 of 6), the largest split count down to 3/4 of
    // it whose clusters can: fewer, longer splits that all start early beat
    // more splits of which one cluster waits for the previous launch to leave.
    // (The workspace is sized for `splits`, an upper bound.)
    if (early >= 2 && !contig && !host_kv && splits > 2 && splits <= kClusterMax) {
        auto fits_twice = [&](int S) {
            const int v = variant_of(S);
            return attn_cluster_fits(d.G, v, S, 2 * d.units(), slots_of(S, v), false);
        };
        if (!fits_twice(splits))
            for (int S = splits - 1; 4 * S >= 3 * splits; --S)
                if (fits_twice(S)) {
                    splits = S;
                    break;
                }
    }
    const int var = variant_of(splits);
    const int slots = slots_of(splits, var);
    const bool cluster = attn_cluster_fits(d.G, var, splits, d.units(), slots, scores_out && hist_out);
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
    a.early = early;
    a.sout = scores_out;
    a.scale = scale;
    a.lse = lse_out;
    a.slots = slots;
    a.hout = scores_out ? hist_out : nullptr;
    dim3 grid(splits, d.units());
    switch (d.G) {
        case 1: e = attn_dispatch<1>(var, cluster, grid, st, a); break;
        case 2: e = attn_dispatch<2>(var, cluster, grid, st, a); break;
        case 4: e = attn_dispatch<4>(var, cluster, grid, st, a); break;
        case 8: e = attn_dispatch<8>(var, cluster, grid, st, a); break;
        default: return cudaErrorInvalidValue;
    }
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa

#ifdef TSA_DEBUG_KNOBS
extern "C" int tsa_debug_attn_skip_tile(int tile) {
    return (int)cudaMemcpyToSymbol(tsa::g_debug_attn_skip_tile, &tile, sizeof tile);
}
#endif
