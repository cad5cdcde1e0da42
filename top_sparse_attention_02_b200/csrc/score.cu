// score.cu -- block mode's step 1: score every block's mean key against the
// current query group, and the block summaries (the means) themselves.  The
// per-token scan of token mode is score_tc.cu.
//
// "inference-time context sparsity: illusion or opportunity?", sec. 2 (oracle
// Top-K): importance is the scaled logit, reduced over the GQA group by max.
// HyLRA sec. 2.4: 128-token blocks, scored through their mean key.
//
// The means are fp32 rows (512 B) and 128x fewer than the keys, so this is a
// short HBM-bound pass that must not run out of CTAs: each warp takes one step
// of rows with coalesced 16-byte loads (a half-warp per row, 8 dims per lane),
// keeps the g query heads of the kv-head in registers, so one read serves the
// whole GQA group, and reduces the per-lane partial dot products with a
// reduce-scatter across the half-warp.
#include "common.cuh"
#include "launch.h"

namespace tsa {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;

template <int G>
__global__ void __launch_bounds__(kScoreThreads)
score_kernel(const __nv_bfloat16* __restrict__ Q, const float* __restrict__ means,
             const int32_t* __restrict__ lens, int Hkv, int Ncap, int rows_cap, int block,
             float scale, float* __restrict__ scores, uint32_t* __restrict__ hist,
             unsigned* __restrict__ flag) {
    constexpr int R = 16 / G;          // rows per half-warp (R*G = 16 partial dots)
    constexpr int kRowsWarp = 2 * R;   // rows per warp
    constexpr int kRowsCta = kRowsWarp * kScoreWarps;
    const int unit = blockIdx.y;
    const int b = unit / Hkv, kvh = unit - b * Hkv;
    griddep_wait();
    griddep_launch();
    int len = lens[b];
    if (len < 0 || len > Ncap) {
        if (threadIdx.x == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    const int n = ceil_div(len, block);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4, c = lane & 15;
    const int base = blockIdx.x * kRowsCta + warp * kRowsWarp;
    if (base >= n) return;

    float q[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const __nv_bfloat16* qp = Q + ((size_t)(b * Hkv + kvh) * G + h) * kD + 8 * c;
        unpack8(*reinterpret_cast<const uint4*>(qp), q[h]);
    }
    const float* kb = means + (size_t)unit * rows_cap * kD;
    uint4 raw[R][2];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int row = base + 2 * r + half;
        const float* p = kb + (size_t)row * kD + 8 * c;
        raw[r][0] = row < n ? ld_stream(p) : make_uint4(0, 0, 0, 0);
        raw[r][1] = row < n ? ld_stream(p + 4) : make_uint4(0, 0, 0, 0);
    }
    float v[16];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float kf[8] = {__uint_as_float(raw[r][0].x), __uint_as_float(raw[r][0].y),
                             __uint_as_float(raw[r][0].z), __uint_as_float(raw[r][0].w),
                             __uint_as_float(raw[r][1].x), __uint_as_float(raw[r][1].y),
                             __uint_as_float(raw[r][1].z), __uint_as_float(raw[r][1].w)};
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) s = fmaf(kf[e], q[h][e], s);
            v[r * G + h] = s;
        }
    }
    // lane c of each half now gets the full dot of (row 2*(c/G)+half, head c%G)
    halfwarp_reduce_scatter16(v, c);
    float m = v[0];
#pragma unroll
    for (int o = 1; o < G; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int row = base + 2 * (c / G) + half;
    // scale > 0, so scale * max_h(z_h) = max_h(scale * z_h) exactly (rounding is monotone)
    if ((c % G) == 0 && row < n) {
        const float v = m * scale;
        scores[(size_t)unit * rows_cap + row] = v;
        // the top-k's first digit (one global atomic per block: 128x fewer than tokens)
        if (hist) atomicAdd(&hist[(size_t)unit * kHistBins + (order_key(v) >> 21)], 1u);
    }
}

// One CTA per (block, unit); thread t owns dimension t and sums the block's
// valid rows in fp32, in row order.
__global__ void __launch_bounds__(kD)
block_mean_kernel(const __nv_bfloat16* __restrict__ K, const int32_t* __restrict__ lens, int Hkv,
                  int Ncap, int NB, int block, float* __restrict__ Kmean, unsigned* __restrict__ flag) {
    const int unit = blockIdx.y, beta = blockIdx.x;
    const int b = unit / Hkv;
    int len = lens[b];
    if (len < 0 || len > Ncap) {
        if (threadIdx.x == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    const int t0 = beta * block;
    if (t0 >= len) return;
    const int t1 = min(t0 + block, len);
    const unsigned short* kb = reinterpret_cast<const unsigned short*>(K) + (size_t)unit * Ncap * kD;
    const int t = threadIdx.x;
    float s = 0.f;
    for (int row = t0; row < t1; ++row) s += __uint_as_float((uint32_t)kb[(size_t)row * kD + t] << 16);
    Kmean[((size_t)unit * NB + beta) * kD + t] = s / (float)(t1 - t0);
}

cudaError_t launch_score(const void* Q, const void* keys, const int32_t* lens, const Dims& d,
                         int block, float scale, float* scores, uint32_t* hist, unsigned* flag,
                         cudaStream_t st, bool early) {
    if (d.units() == 0 || d.Ncap == 0) return cudaSuccess;
    if (block == 1) return launch_score_tc(Q, keys, lens, d, scale, scores, hist, flag, st, early);
    const int rows_cap = rows_cap_of(d, block);
    const int rows_cta = 2 * (16 / d.G) * kScoreWarps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ceil_div(rows_cap, rows_cta), d.units());
    cfg.blockDim = dim3(kScoreThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
    const float* m = static_cast<const float*>(keys);
    cudaError_t e;
    switch (d.G) {
        case 1: e = cudaLaunchKernelEx(&cfg, score_kernel<1>, q, m, lens, d.Hkv, d.Ncap, rows_cap, block, scale, scores, hist, flag); break;
        case 2: e = cudaLaunchKernelEx(&cfg, score_kernel<2>, q, m, lens, d.Hkv, d.Ncap, rows_cap, block, scale, scores, hist, flag); break;
        case 4: e = cudaLaunchKernelEx(&cfg, score_kernel<4>, q, m, lens, d.Hkv, d.Ncap, rows_cap, block, scale, scores, hist, flag); break;
        case 8: e = cudaLaunchKernelEx(&cfg, score_kernel<8>, q, m, lens, d.Hkv, d.Ncap, rows_cap, block, scale, scores, hist, flag); break;
        default: return cudaErrorInvalidValue;
    }
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_block_summarize(const void* K, const int32_t* lens, const Dims& d, int block,
                                   float* Kmean, unsigned* flag, cudaStream_t st) {
    if (d.units() == 0 || d.Ncap == 0) return cudaSuccess;
    const int NB = ceil_div(d.Ncap, block);
    dim3 grid(NB, d.units());
    block_mean_kernel<<<grid, kD, 0, st>>>(static_cast<const __nv_bfloat16*>(K), lens, d.Hkv,
                                           d.Ncap, NB, block, Kmean, flag);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tsa
