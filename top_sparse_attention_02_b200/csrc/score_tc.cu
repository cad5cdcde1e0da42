// score_tc.cu -- step 1 of the decode path on the 5th-generation tensor cores:
// the group product S = K Q^T ([rows x 128] . [128 x heads]) of every cached key
// against the kv-head's query group, then the max over the group's heads.
//
// "inference-time context sparsity: illusion or opportunity?", sec. 2 (oracle
// Top-K: importance of every token, chosen exactly); "Flash Attention vs
// Sparse Attention", DSA stage 1 (one pass over the whole context).
//
// Why tensor cores here: the scan is HBM-bound (every K byte read once), but the
// CUDA-core version spends ~36 warp instructions per 256-byte row on
// bf16 unpacking, FMAs and the cross-lane reduction, and ncu showed it
// latency/issue-bound at 57-69% of HBM bandwidth.  On tcgen05 the whole
// [128 rows x 128] x [128 x 16] tile is 8 MMA instructions from one thread.
//
// Design (per CTA: one unit, a range of 128-row tiles; 6 warps):
//   warp 0  TMA producer: 2-D tensor loads (box 64 dims x 128 rows, 128-byte
//           swizzle) of K into a 2-stage shared-memory ring, completing on
//           "full" mbarriers;
//   warp 1  MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 accumulate),
//           M = 128 rows, N = 16 (the g <= 8 query heads, zero-padded),
//           K = 16 x 8 steps, into one of two TMEM accumulators; tcgen05.commit
//           frees the ring stage and publishes the accumulator;
//   warps 2-5 epilogue: tcgen05.ld of their 32 TMEM lanes (= rows), max over the
//           g heads, times the scale, coalesced store of the scores; when asked,
//           also a shared-memory histogram of the scores' top 11 key bits,
//           added into the unit's histogram at the end (the top-k's first
//           digit, counted here where the ALUs idle behind HBM).
// Q is written once per CTA into shared memory in the same swizzled K-major
// layout (the B operand).  Every mbarrier wait is bounded: on expiry the kernel
// raises the device timeout flag and each role stops; before the CTA leaves,
// the producer waits (bounded) for the tile loads it issued and the MMA issuer
// for the MMAs it issued, so that nothing lands in shared memory or TMEM after
// TMEM is freed and the CTA is gone.  The scores are then unspecified.
//
// With `early` (the caller's promise that the kernel before this one on the
// stream writes neither the lengths nor K), the first two K tiles are requested
// before waiting on that kernel (programmatic dependent launch), so the scan's
// first loads overlap its end; Q, the scores and the histogram are touched only
// after the wait.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"

namespace tsa {

constexpr int kTcThreads = 192;         // 6 warps
constexpr int kTcTileRows = 128;        // M
constexpr int kTcN = 16;                // N: query heads padded to 16
constexpr int kTcStages = 2;  // 2 x 32 KB in flight per CTA, 2 CTAs per SM (measured: 2 >= 3 > 4)
constexpr int kTcHalfBytes = kTcTileRows * 128;       // 64 dims x 128 rows x 2 B = 16 KB
constexpr int kTcStageBytes = 2 * kTcHalfBytes;       // the full 128-dim tile: 32 KB
constexpr int kTcQHalfBytes = kTcN * 128;             // 16 rows x 128 B = 2 KB
constexpr int kTcTilesPerCta = 32;                    // 4096 rows per CTA (the 128K scan: 256 CTAs, one wave)
constexpr int kTcSms = 148;
constexpr int kTcSmem = 1024 /*align slack*/ + kTcStages * kTcStageBytes + 2 * kTcQHalfBytes;
#ifndef TSA_WAIT_SPINS
constexpr long kTcSpins = 1L << 22;
#else
constexpr long kTcSpins = TSA_WAIT_SPINS;  // a debug build's short limit
#endif

#ifdef TSA_DEBUG_KNOBS
// Debug build only (never in the product library): the tile (of CTA (0, 0))
// whose load the producer leaves out, so that the waits on it run out; -1: none.
__device__ int g_debug_skip_tile = -1;
#endif
// instruction descriptor: D f32 (bits 4-5 = 1), A bf16 (7-9 = 1), B bf16 (10-12 = 1),
// both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28
constexpr uint32_t kTcIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcN >> 3) << 17) |
                              ((uint32_t)(kTcTileRows >> 4) << 24);

__device__ __forceinline__ unsigned su32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }

// shared-memory matrix descriptor: 128-byte swizzle, K-major, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t sw128_desc(unsigned saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) /* LBO (unused) */ |
           ((uint64_t)(1024 >> 4) << 32) /* SBO */ | ((uint64_t)1 << 46) /* version */ |
           ((uint64_t)2 << 61) /* SWIZZLE_128B */;
}

__device__ __forceinline__ void tc_mbar_init(unsigned bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void tc_arrive(unsigned bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_arrive_tx(unsigned bar, unsigned bytes) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}
// bounded wait for the phase of the given parity; false = gave up (flag raised,
// unless flag is NULL: a drain wait at the end)
__device__ __forceinline__ bool tc_wait(unsigned bar, unsigned parity, unsigned* flag) {
    for (long i = 0; i < kTcSpins; ++i) {
        unsigned done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    if (flag) atomicOr(flag, kFlagTimeout);
    return false;
}

template <int G>
__global__ void __launch_bounds__(kTcThreads, 2)
score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __nv_bfloat16* __restrict__ Q,
                const int32_t* __restrict__ lens, int Hkv, int Ncap, float scale,
                float* __restrict__ scores, uint32_t* __restrict__ hist, int tiles_per_cta,
                unsigned* __restrict__ flag, int early) {
    extern __shared__ unsigned char tc_smem_raw[];
    __shared__ __align__(8) uint64_t s_full[kTcStages], s_empty[kTcStages], s_tfull[2], s_tempty[2];
    __shared__ uint32_t s_tmem;
    __shared__ uint32_t s_hist[kHistBins];  // this CTA's counts of the keys' top digit (when hist != NULL)

    const int unit = blockIdx.y;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (!early) griddep_wait();
    int len = early ? __ldcg(lens + b) : lens[b];
    if (len < 0 || len > Ncap) {
        if (tid == 0 && blockIdx.x == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    const int ntiles_unit = ceil_div(len, kTcTileRows);
    const int t0 = blockIdx.x * tiles_per_cta;
    const int t1 = min(t0 + tiles_per_cta, ntiles_unit);
    if (t0 >= t1) return;  // uniform: before any barrier or TMEM use
    const int nt = t1 - t0;

    // 1024-byte aligned carve-up: [stage 0: half0 | half1][stage 1]...[Q half0 | Q half1]
    const unsigned raw = su32(tc_smem_raw);
    const unsigned base = (raw + 1023u) & ~1023u;
    unsigned char* basep = tc_smem_raw + (base - raw);
    const unsigned qbase = base + kTcStages * kTcStageBytes;

    // ---- set-up: barriers (thread 0), TMEM (warp 1), Q as the swizzled B operand (warps 2-5)
    if (hist)
        for (int i = tid; i < kHistBins; i += kTcThreads) s_hist[i] = 0u;
    if (tid == 0) {
        for (int i = 0; i < kTcStages; ++i) {
            tc_mbar_init(su32(&s_full[i]), 1);
            tc_mbar_init(su32(&s_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc_mbar_init(su32(&s_tfull[i]), 1);
            tc_mbar_init(su32(&s_tempty[i]), 128);
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 1) {  // 32 columns: two 16-column accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(su32(&s_tmem)),
                     "r"(32)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    // ---- the producer's tile loads (warp 0, lane 0)
    const int row_base = unit * Ncap;
    // K is read once: evict it from L2 first, so the scores (kept with
    // evict_last below) are still there when the top-k reads them
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
    auto issue = [&](int i) {
        const int s = i % kTcStages;
        const unsigned full = su32(&s_full[s]);
#ifdef TSA_DEBUG_KNOBS
        if (i == g_debug_skip_tile && blockIdx.x == 0 && unit == 0) return;  // neither armed nor loaded
#endif
        tc_arrive_tx(full, kTcStageBytes);
        const int y = row_base + (t0 + i) * kTcTileRows;
        const unsigned dst = base + s * kTcStageBytes;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            asm volatile(
                "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;\n" ::"r"(
                    dst + half * kTcHalfBytes),
                "l"(&kmap), "r"(half * 64), "r"(y), "r"(full), "l"(pol)
                : "memory");
        }
    };
    int issued = 0;  // warp 0, lane 0: tiles requested so far
    if (early) {
        if (tid >= 64 && tid < 64 + 2 * G) prefetch_l2(Q + (size_t)unit * G * kD + (tid - 64) * 64);  // Q into L2
        // the first stages' loads before waiting on the previous kernel
        __syncthreads();  // the barriers are initialised
        if (warp == 0 && lane == 0)
            for (; issued < nt && issued < kTcStages; ++issued) issue(issued);
        griddep_wait();
    }
    if (warp >= 2) {  // Q rows n < G (bf16 as stored), rows G..15 zero; 16-byte chunks swizzled
        const int t = tid - 64;  // 0..127: (row n, 16-byte chunk c of the 256-byte row)
        const int n = t >> 3, c16 = t & 7;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (n < G) v = *reinterpret_cast<const uint4*>(Q + ((size_t)unit * G + n) * kD + half * 64 + c16 * 8);
            unsigned char* dst = basep + (qbase - base) + half * kTcQHalfBytes + n * 128 + ((c16 ^ (n & 7)) << 4);
            *reinterpret_cast<uint4*>(dst) = v;
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // generic writes -> tensor-core reads
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // ---- TMA producer
        if (lane == 0) {
            for (; issued < nt; ++issued) {
                const int i = issued, s = i % kTcStages;
                if (i >= kTcStages && !tc_wait(su32(&s_empty[s]), (unsigned)((i / kTcStages) - 1) & 1u, flag)) break;
                issue(i);
            }
            // the last load of each stage has landed (at once, unless a wait
            // gave up): none may land after the CTA has gone
            for (int j = max(0, issued - kTcStages); j < issued; ++j)
                tc_wait(su32(&s_full[j % kTcStages]), (unsigned)(j / kTcStages) & 1u, nullptr);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0) {
            int done = 0;  // tiles whose MMAs were issued
            for (int i = 0; i < nt; ++i) {
                const int s = i % kTcStages, bsel = i & 1;
                if (!tc_wait(su32(&s_full[s]), (unsigned)(i / kTcStages) & 1u, flag)) break;
                if (i >= 2 && !tc_wait(su32(&s_tempty[bsel]), (unsigned)((i >> 1) - 1) & 1u, flag)) break;
                asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
                const uint32_t d = tmem + (uint32_t)(bsel * kTcN);
                const unsigned abase = base + s * kTcStageBytes;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int half = k >> 2, kk = k & 3;
                    const uint64_t ad = sw128_desc(abase + half * kTcHalfBytes + kk * 32);
                    const uint64_t bd = sw128_desc(qbase + half * kTcQHalfBytes + kk * 32);
                    asm volatile(
                        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
                        "l"(ad), "l"(bd), "r"(kTcIdesc), "r"(k)
                        : "memory");
                }
                // both arrive when the MMAs above complete
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                                 su32(&s_empty[s]))
                             : "memory");
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                                 su32(&s_tfull[bsel]))
                             : "memory");
                done = i + 1;
            }
            // the last MMAs issued have completed (their commit freed the ring
            // stage) before TMEM is freed below
            if (done > 0) {
                const int j = done - 1;
                tc_wait(su32(&s_empty[j % kTcStages]), (unsigned)(j / kTcStages) & 1u, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp quarter q reads TMEM lanes 32q..32q+31 (tile rows)
        const int q = warp & 3;
        float* out = scores + (size_t)unit * Ncap;
        uint64_t keep;  // the scores are read again right after this kernel: keep them in L2
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\n" : "=l"(keep));
        for (int i = 0; i < nt; ++i) {
            const int bsel = i & 1;
            // every lane waits itself; the warp goes on only if all saw the
            // accumulator (tcgen05.ld below is warp-collective), else it stops
            const bool ok = __all_sync(0xffffffffu, tc_wait(su32(&s_tfull[bsel]), (unsigned)(i >> 1) & 1u, flag));
            if (!ok) break;
            asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
            uint32_t r[16];
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(bsel * kTcN);
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                "%13, %14, %15}, [%16];\n"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                  "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                  "=r"(r[15])
                : "r"(taddr)
                : "memory");
            asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
            float m = __uint_as_float(r[0]);
#pragma unroll
            for (int h = 1; h < G; ++h) m = fmaxf(m, __uint_as_float(r[h]));
            const int row = (t0 + i) * kTcTileRows + q * 32 + lane;
            // scale > 0, so scale * max_h(z_h) = max_h(scale * z_h) exactly (rounding is monotone)
            if (row < len) {
                const float v = m * scale;
                asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;\n" ::"l"(out + row), "f"(v), "l"(keep)
                             : "memory");
                if (hist) atomicAdd(&s_hist[order_key(v) >> 21], 1u);
            }
            asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
            tc_arrive(su32(&s_tempty[bsel]));
        }
    }
    griddep_launch();
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(32) : "memory");
    }
    // this CTA's top-digit counts into the unit's histogram (the dependent top-k
    // reads it only once this grid has completed)
    if (hist) {
        uint32_t* hu = hist + (size_t)unit * kHistBins;
        for (int i = tid; i < kHistBins; i += kTcThreads)
            if (const uint32_t c = s_hist[i]) atomicAdd(&hu[i], c);
    }
}

// ---- host: tensor map over K viewed as [B*Hkv*Ncap rows] x [128 dims] bf16
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

static cudaError_t get_encode() {
    if (g_encode) return cudaSuccess;
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return cudaSuccess;
}

static int g_tc_configured[64];

cudaError_t launch_score_tc(const void* Q, const void* K, const int32_t* lens, const Dims& d, float scale,
                            float* scores, uint32_t* hist, unsigned* flag, cudaStream_t st, bool early) {
    if (d.units() == 0 || d.Ncap == 0) return cudaSuccess;
    cudaError_t e = get_encode();
    if (e != cudaSuccess) return e;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)d.units() * (cuuint64_t)d.Ncap};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTcTileRows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(K), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !g_tc_configured[dev]) {
        const void* fns[4] = {(const void*)score_tc_kernel<1>, (const void*)score_tc_kernel<2>,
                              (const void*)score_tc_kernel<4>, (const void*)score_tc_kernel<8>};
        for (const void* f : fns) {
            e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
            if (e != cudaSuccess) return e;
        }
        g_tc_configured[dev] = 1;
    }
    // 32 tiles a CTA, unless that leaves SMs idle (short or few units): then
    // about two CTAs per SM
    const int tiles = ceil_div(d.Ncap, kTcTileRows);
    int per = kTcTilesPerCta;
    if ((long long)d.units() * ceil_div(tiles, per) < kTcSms)
        per = max(1, ceil_div(tiles * d.units(), 2 * kTcSms));
    dim3 grid(ceil_div(tiles, per), d.units());
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = kTcSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    switch (d.G) {
        case 1: e = cudaLaunchKernelEx(&cfg, score_tc_kernel<1>, map, q, lens, d.Hkv, d.Ncap, scale, scores, hist, per, flag, early ? 1 : 0); break;
        case 2: e = cudaLaunchKernelEx(&cfg, score_tc_kernel<2>, map, q, lens, d.Hkv, d.Ncap, scale, scores, hist, per, flag, early ? 1 : 0); break;
        case 4: e = cudaLaunchKernelEx(&cfg, score_tc_kernel<4>, map, q, lens, d.Hkv, d.Ncap, scale, scores, hist, per, flag, early ? 1 : 0); break;
        case 8: e = cudaLaunchKernelEx(&cfg, score_tc_kernel<8>, map, q, lens, d.Hkv, d.Ncap, scale, scores, hist, per, flag, early ? 1 : 0); break;
        default: return cudaErrorInvalidValue;
    }
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa

#ifdef TSA_DEBUG_KNOBS
// Debug build only: which tile's load the scorer (0) or the attention's
// contiguous-tile path (1) leaves out in CTA (0, 0); -1 for none.  Returns a
// cudaError_t.
extern "C" int tsa_debug_attn_skip_tile(int tile);
extern "C" int tsa_debug_skip_tile(int which, int tile) {
    if (which == 1) return tsa_debug_attn_skip_tile(tile);
    return (int)cudaMemcpyToSymbol(tsa::g_debug_skip_tile, &tile, sizeof tile);
}
#endif
