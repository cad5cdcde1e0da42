// topk.cu -- step 2 of the decode path: exact top-k per (sequence, kv-head).
//
// "inference-time context sparsity: illusion or opportunity?", sec. 2: oracle
// Top-K picks exactly the k highest-scoring tokens.  Ties go to the lower
// index and the output is in ascending index order, so the result is unique.
//
// Design (B200): one thread-block cluster of C CTAs per unit.  Each CTA holds
// its slice of the unit's scores in shared memory as order-preserving 32-bit
// keys, so the scores are read from L2/HBM once.  A radix select with 11/11/10
// bit digits finds the k-th largest key T exactly: per pass every CTA builds a
// shared-memory histogram of the keys still in play, the cluster reads all C
// histograms through distributed shared memory, and a block-wide scan from the
// top bin finds the digit of T.  Then an ordered compaction: keys > T are all
// taken, keys == T are taken in index order until k is reached; each warp walks
// its segment 32 keys at a time with ballots, and CTA offsets come from a scan
// over the cluster.  Cluster barriers are hardware barriers; there is no
// software spin anywhere in this kernel.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace tsa {

constexpr int kTkThreads = 1024;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkLocalPref = 16384;  // keys per CTA before the cluster grows (64 KB)
constexpr int kTkLocalMax = 40960;   // hard cap per CTA (160 KB of keys)
constexpr int kTkHist = 2048;

// Exclusive scan over the 1024 threads of the block; *total gets the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t* wsum, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = wsum[lane];
        uint32_t winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += y;
        }
        wsum[lane] = winc - w;
        if (lane == 31) wsum[32] = winc;
    }
    __syncthreads();
    const uint32_t ex = wsum[warp] + inc - x;
    *total = wsum[32];
    __syncthreads();
    return ex;
}

__global__ void __launch_bounds__(kTkThreads, 1)
topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ lens,
            const int32_t* __restrict__ kreq, int k_max, int Hkv, int Ncap, int rows_cap, int block,
            int chunk, int32_t* __restrict__ idx, unsigned* __restrict__ flag) {
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int unit = blockIdx.x / C;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    extern __shared__ __align__(16) uint32_t tk_smem[];
    uint32_t* keys = tk_smem;          // [chunk]
    uint32_t* hist = tk_smem + chunk;  // [2][kTkHist], double-buffered across passes
    __shared__ uint32_t wsum[33];
    __shared__ uint32_t s_sel[2];
    __shared__ uint32_t s_ctatot[2];   // this CTA's (gt, eq) totals, read by later ranks
    __shared__ uint32_t s_warpbase[kTkWarps][2];
    __shared__ uint32_t s_base[2];

    int len = lens[b];
    if (len < 0 || len > Ncap) {
        if (tid == 0 && rank == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    const int n = block == 1 ? len : ceil_div(len, block);
    int kb = kreq ? kreq[b] : k_max;
    if (kb < 0) kb = 0;
    if (kb > n) kb = n;
    if (kb > k_max) {
        if (tid == 0 && rank == 0) atomicOr(flag, kFlagBounds);
        kb = k_max;
    }
    int32_t* out = idx + (size_t)unit * k_max;
    const int lo = rank * chunk;
    const int nloc = max(0, min(chunk, n - lo));

    // Degenerate units need no selection; every CTA of the cluster takes the
    // same branch, so no cluster barrier is left waiting.
    if (kb == 0 || kb == n) {
        for (int i = tid; i < nloc; i += kTkThreads)
            if (lo + i < kb) out[lo + i] = lo + i;
        if (rank == 0)
            for (int p = kb + tid; p < k_max; p += kTkThreads) out[p] = -1;
        return;
    }

    const float* su = scores + (size_t)unit * rows_cap + lo;
    for (int i0 = tid; i0 < nloc; i0 += 8 * kTkThreads) {  // 8 independent loads in flight
        float f[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kTkThreads;
            f[j] = i < nloc ? __ldcg(su + i) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * kTkThreads;
            if (i < nloc) keys[i] = order_key(f[j]);
        }
    }

    // ---- radix select of the k-th largest key: digits [31:21], [20:10], [9:0]
    uint32_t prefix = 0, pmask = 0, krem = (uint32_t)kb;
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
        const int nbins = p == 2 ? 1024 : 2048;
        const uint32_t dmask = (uint32_t)nbins - 1u;
        uint32_t* h = hist + (p & 1) * kTkHist;
        for (int i = tid; i < kTkHist; i += kTkThreads) h[i] = 0u;
        __syncthreads();
        for (int i = tid; i < nloc; i += kTkThreads) {
            const uint32_t k = keys[i];
            if ((k & pmask) == prefix) atomicAdd(&h[(k >> shift) & dmask], 1u);
        }
        cluster.sync();  // all C histograms of this pass are complete
        // thread t owns bins nbins-1-2t and nbins-2-2t: ascending t = descending bins
        const int hb0 = nbins - 1 - 2 * tid, hb1 = hb0 - 1;
        uint32_t c0 = 0, c1 = 0;
        if (hb1 >= 0) {
#pragma unroll 4
            for (int r = 0; r < C; ++r) {
                const uint32_t* rh = cluster.map_shared_rank(h, r);
                c0 += rh[hb0];
                c1 += rh[hb1];
            }
        }
        uint32_t total;
        const uint32_t above = block_excl_scan(c0 + c1, wsum, &total);
        if (hb1 >= 0 && above < krem && krem <= above + c0 + c1) {  // exactly one thread
            if (krem <= above + c0) {
                s_sel[0] = (uint32_t)hb0;
                s_sel[1] = above;
            } else {
                s_sel[0] = (uint32_t)hb1;
                s_sel[1] = above + c0;
            }
        }
        __syncthreads();
        prefix |= s_sel[0] << shift;
        pmask |= dmask << shift;
        krem -= s_sel[1];
        __syncthreads();
    }
    const uint32_t T = prefix;  // the k-th largest key; krem keys equal to T are taken

    // ---- ordered compaction.  Warp w walks segment [w*seg, (w+1)*seg) of the slice.
    const int seg = ceil_div(ceil_div(nloc, kTkWarps), 32) * 32;
    const int wbeg = min(warp * seg, nloc), wend = min(wbeg + seg, nloc);
    uint32_t wgt = 0, weq = 0;
    for (int i0 = wbeg; i0 < wend; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < wend ? keys[i] : 0u;
        wgt += __popc(__ballot_sync(0xffffffffu, i < wend && k > T));
        weq += __popc(__ballot_sync(0xffffffffu, i < wend && k == T));
    }
    if (lane == 0) {
        s_warpbase[warp][0] = wgt;
        s_warpbase[warp][1] = weq;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the 32 warp totals, both counters
        const uint32_t g = s_warpbase[lane][0], e = s_warpbase[lane][1];
        uint32_t gi = g, ei = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t yg = __shfl_up_sync(0xffffffffu, gi, o);
            const uint32_t ye = __shfl_up_sync(0xffffffffu, ei, o);
            if (lane >= o) {
                gi += yg;
                ei += ye;
            }
        }
        s_warpbase[lane][0] = gi - g;
        s_warpbase[lane][1] = ei - e;
        if (lane == 31) {
            s_ctatot[0] = gi;
            s_ctatot[1] = ei;
        }
    }
    cluster.sync();  // CTA totals visible cluster-wide
    if (warp == 0) {
        uint32_t g = 0, e = 0;
        if (lane < rank) {
            const uint32_t* rt = cluster.map_shared_rank(s_ctatot, lane);
            g = rt[0];
            e = rt[1];
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane == 0) {
            s_base[0] = g;
            s_base[1] = e;
        }
    }
    __syncthreads();
    uint32_t gb = s_base[0] + s_warpbase[warp][0];  // keys > T before this warp's next round
    uint32_t eb = s_base[1] + s_warpbase[warp][1];  // keys == T before it
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int i0 = wbeg; i0 < wend; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < wend ? keys[i] : 0u;
        const bool isg = i < wend && k > T, ise = i < wend && k == T;
        const uint32_t bg = __ballot_sync(0xffffffffu, isg), be = __ballot_sync(0xffffffffu, ise);
        const uint32_t my_g = gb + __popc(bg & lt_mask), my_e = eb + __popc(be & lt_mask);
        const bool take = isg || (ise && my_e < krem);
        const uint32_t pos = isg ? my_g + min(my_e, krem) : my_g + my_e;
        if (take) {
            if (pos < (uint32_t)kb) out[pos] = lo + i;
            else atomicOr(flag, kFlagBounds);  // unreachable when the select is consistent
        }
        gb += __popc(bg);
        eb += __popc(be);
    }
    if (rank == 0)
        for (int p = kb + tid; p < k_max; p += kTkThreads) out[p] = -1;
    cluster.sync();  // no CTA leaves while another may still read its shared memory
}

bool topk_plan(int rows_cap, int* cluster, int* chunk) {
    int C = 1;
    while (C < 16 && ceil_div(rows_cap, C) > kTkLocalPref) C *= 2;
    int ch = ceil_div(rows_cap, C);
    ch = ceil_div(ch, 32) * 32;
    if (ch < 32) ch = 32;
    if (ch > kTkLocalMax) return false;
    *cluster = C;
    *chunk = ch;
    return true;
}

static int g_tk_configured[64];

cudaError_t launch_topk(const float* scores, const int32_t* lens, const int32_t* kreq, int k_max,
                        const Dims& d, int block, int32_t* idx, unsigned* flag, cudaStream_t st) {
    if (d.units() == 0 || k_max == 0) return cudaSuccess;
    const int rows_cap = rows_cap_of(d, block);
    int C = 1, chunk = 32;
    if (!topk_plan(rows_cap, &C, &chunk)) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !g_tk_configured[dev]) {
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (kTkLocalMax + 2 * kTkHist) * (int)sizeof(uint32_t));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        g_tk_configured[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(d.units() * C));
    cfg.blockDim = dim3(kTkThreads);
    cfg.dynamicSmemBytes = (size_t)(chunk + 2 * kTkHist) * sizeof(uint32_t);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, topk_kernel, scores, lens, kreq, k_max, d.Hkv, d.Ncap, rows_cap,
                           block, chunk, idx, flag);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa
