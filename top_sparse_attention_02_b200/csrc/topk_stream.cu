// topk_stream.cu -- step 2 of the decode path for many short units: exact top-k
// per (sequence, kv-head) with one CTA per unit and no cluster.
//
// "inference-time context sparsity: illusion or opportunity?", sec. 2: oracle
// Top-K picks exactly the k highest-scoring tokens.  Ties go to the lower
// index and the output is in ascending index order, so the result is unique.
//
// When a batch has many units (hundreds of sequences x kv-heads, a few
// thousand to tens of thousands of rows each) the cluster kernel of topk.cu
// spends its time in barriers and runs in several waves (its keys live in
// ~180 KB of shared memory).  Here a unit is one CTA whose warps each own a
// contiguous run of the unit's scores, streamed from L2 with 16 loads in
// flight per lane; only the keys that can still be selected are kept, in index
// order, in a small per-warp list in shared memory:
//   digit 1 (top 11 bits of the order-preserving key): the scorer's histogram
//           when the decode step provides one (then zeroed for the next step),
//           else one streaming pass of shared-memory atomics; a block scan
//           from the top finds the bin d0 of the k-th largest key and the exact
//           number of keys at or above it;
//   filter: one streaming pass keeps the keys whose top digit is >= d0 (ballot
//           compaction, so each warp's list stays in index order);
//   digits 2, 3 (11 and 10 bits): histograms over the list find T, the k-th
//           largest key, and krem, the number of keys equal to T to take;
//   output: keys > T and the first krem keys == T, their positions from a
//           ballot count per warp and a scan over the warps.
// If the list would overflow (heavy ties, or k near the unit's length) every
// later step streams the unit's scores again instead of walking the list.
#include "common.cuh"
#include "launch.h"

namespace tsa {

constexpr int kTsNB = 16;  // loads in flight per lane while streaming

template <int THREADS>
__device__ __forceinline__ uint32_t ts_block_scan(uint32_t x, uint32_t* wsum, uint32_t* total) {
    constexpr int W = THREADS / 32;
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
        const uint32_t w = lane < W ? wsum[lane] : 0u;
        uint32_t winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += y;
        }
        if (lane < W) wsum[lane] = winc - w;
        if (lane == 31) wsum[32] = winc;
    }
    __syncthreads();
    const uint32_t ex = wsum[warp] + inc - x;
    *total = wsum[32];
    __syncthreads();
    return ex;
}

// 256 threads: at most 64 registers, so that 4 CTAs (units) share an SM
template <int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS <= 256 ? 4 : 1)
topk_stream_kernel(const float* __restrict__ scores, const int32_t* __restrict__ lens,
                   const int32_t* __restrict__ kreq, int k_max, int Hkv, int Ncap, int rows_cap, int block,
                   int wcap, int32_t* __restrict__ idx, uint32_t* __restrict__ hist,
                   unsigned* __restrict__ flag) {
    constexpr int W = THREADS / 32;
    extern __shared__ uint32_t ts_list[];  // [W][wcap] keys, then [W][wcap] row indices
    __shared__ __align__(16) uint32_t h[kHistBins];
    __shared__ uint32_t wsum[33];
    __shared__ uint32_t s_sel[2];
    __shared__ uint32_t s_cnt[W];        // entries in each warp's list
    __shared__ uint32_t s_off[W][2];     // per-warp (gt, eq) counts, then their exclusive offsets
    __shared__ int s_over;

    const int unit = blockIdx.x;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_wait();
    griddep_launch();

    int len = lens[b];
    if (len < 0 || len > Ncap) {
        if (tid == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    const int n = block == 1 ? len : ceil_div(len, block);
    int kb = kreq ? kreq[b] : k_max;
    if (kb < 0) kb = 0;
    if (kb > n) kb = n;
    if (kb > k_max) {
        if (tid == 0) atomicOr(flag, kFlagBounds);
        kb = k_max;
    }
    int32_t* out = idx + (size_t)unit * k_max;
    uint32_t* hu = hist ? hist + (size_t)unit * kHistBins : nullptr;
    if (kb == 0 || kb == n) {  // nothing to select: the first kb rows, then -1
        for (int p = tid; p < k_max; p += THREADS) out[p] = p < kb ? p : -1;
        if (hu)
            for (int i = tid; i < kHistBins; i += THREADS) hu[i] = 0u;
        return;
    }

    const float* su = scores + (size_t)unit * rows_cap;
    // warp w owns rows [wb, we) of the unit, walked 32 consecutive rows at a time
    const int seg = ceil_div(ceil_div(n, W), 32) * 32;
    const int wb = min(warp * seg, n), we = min(wb + seg, n);
    // f(row, key, valid) for every row of this warp's run, the whole warp together
    auto stream = [&](auto&& f) {
        for (int base = wb; base < we; base += 32 * kTsNB) {
            float v[kTsNB];
#pragma unroll
            for (int j = 0; j < kTsNB; ++j) {
                const int i = base + j * 32 + lane;
                v[j] = i < we ? __ldcg(su + i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < kTsNB; ++j) {
                const int i = base + j * 32 + lane;
                f(i, order_key(v[j]), i < we);
            }
        }
    };
    // from the top bin down, the bin holding the kr-th largest key -> s_sel = (bin, keys above it)
    auto select_bin = [&](int nbins, uint32_t kr) {
        constexpr int kMaxPer = kHistBins / THREADS > 0 ? kHistBins / THREADS : 1;
        const int per = nbins / THREADS > 0 ? nbins / THREADS : 1;
        const int top = nbins - 1 - per * tid;  // bins top, top-1, ..., top-per+1
        uint32_t c[kMaxPer];
        uint32_t sum = 0;
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            c[q] = (q < per && top - q >= 0) ? h[top - q] : 0u;
            sum += c[q];
        }
        uint32_t total;
        uint32_t acc = ts_block_scan<THREADS>(sum, wsum, &total);
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            if (q < per && top - q >= 0 && acc < kr && kr <= acc + c[q]) {  // exactly one (thread, q)
                s_sel[0] = (uint32_t)(top - q);
                s_sel[1] = acc;
            }
            acc += c[q];
        }
        __syncthreads();
    };
    auto clear_hist = [&]() {
        for (int i = tid; i < kHistBins; i += THREADS) h[i] = 0u;
        __syncthreads();
    };

    // ---- digit 1
    if (tid == 0) s_over = 0;
    if (hu) {
        for (int i = tid; i < kHistBins / 4; i += THREADS)
            reinterpret_cast<uint4*>(h)[i] = __ldcg(reinterpret_cast<const uint4*>(hu) + i);
        __syncthreads();
        for (int i = tid; i < kHistBins; i += THREADS) hu[i] = 0u;  // consumed: ready for the next step
    } else {
        clear_hist();
        stream([&](int, uint32_t k, bool v) {
            if (v) atomicAdd(&h[k >> 21], 1u);
        });
        __syncthreads();
    }
    select_bin(kHistBins, (uint32_t)kb);
    const uint32_t d0 = s_sel[0];
    uint32_t krem = (uint32_t)kb - s_sel[1];
    const uint32_t kept = s_sel[1] + h[d0];  // keys whose top digit is >= d0, exactly
    const uint32_t lt = (1u << lane) - 1u;

    // ---- filter into the per-warp lists (index order within each warp).  Most
    // keys fail, so each 32 rows are first tested as raw floats against the
    // smallest float whose key reaches digit d0 (the key order is the float
    // order, -0 = +0; NaN passes and is sorted out by its key), one vote each.
    uint32_t* lkey = ts_list + warp * wcap;
    uint32_t* lrow = ts_list + W * wcap + warp * wcap;
    bool list_mode = kept <= (uint32_t)(W * wcap);
    if (list_mode) {
        const uint32_t kthr = d0 << 21;
        const float fthr = __uint_as_float((kthr & 0x80000000u) ? (kthr & 0x7fffffffu) : ~kthr);
        uint32_t cnt = 0;
        for (int base = wb; base < we; base += 32 * kTsNB) {
            float v[kTsNB];
#pragma unroll
            for (int j = 0; j < kTsNB; ++j) {
                const int i = base + j * 32 + lane;
                v[j] = i < we ? __ldcg(su + i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < kTsNB; ++j) {
                const int i = base + j * 32 + lane;
                // one vote per 32 rows: with k a fraction of a percent of the rows,
                // most steps have no candidate and end here
                const bool maybe = i < we && !(v[j] < fthr);
                if (__ballot_sync(0xffffffffu, maybe) == 0u) continue;
                const uint32_t k = order_key(v[j]);
                const bool keep = maybe && (k >> 21) >= d0;
                const uint32_t bal = __ballot_sync(0xffffffffu, keep);
                const uint32_t pos = cnt + __popc(bal & lt);
                if (keep && pos < (uint32_t)wcap) {
                    lkey[pos] = k;
                    lrow[pos] = (uint32_t)i;
                }
                cnt += __popc(bal);
            }
        }
        if (lane == 0) {
            s_cnt[warp] = cnt;
            if (cnt > (uint32_t)wcap) s_over = 1;
        }
        __syncthreads();
        list_mode = s_over == 0;
    }
    const uint32_t my_cnt = list_mode ? s_cnt[warp] : 0u;
    // f(row, key, valid) over the keys still in play: this warp's list, or its whole run
    auto walk = [&](auto&& f) {
        if (list_mode) {
            for (uint32_t e0 = 0; e0 < my_cnt; e0 += 32) {
                const uint32_t e = e0 + lane;
                const bool v = e < my_cnt;
                f(v ? (int)lrow[e] : 0, v ? lkey[e] : 0u, v);
            }
        } else {
            stream(f);
        }
    };

    // ---- digits 2 and 3
    uint32_t pre = d0 << 21, pm = 0x7ffu << 21;
#pragma unroll 1
    for (int p = 1; p < 3; ++p) {
        const int shift = p == 1 ? 10 : 0;
        const int nbins = p == 1 ? 2048 : 1024;
        const uint32_t dmask = (uint32_t)nbins - 1u;
        clear_hist();
        walk([&](int, uint32_t k, bool v) {
            if (v && (k & pm) == pre) atomicAdd(&h[(k >> shift) & dmask], 1u);
        });
        __syncthreads();
        select_bin(nbins, krem);
        pre |= s_sel[0] << shift;
        pm |= dmask << shift;
        krem -= s_sel[1];
    }
    const uint32_t T = pre;  // the k-th largest key; krem keys equal to T are taken

    // ---- output positions: counts per warp, scan over the warps, then the writes
    uint32_t g_w = 0, e_w = 0;
    walk([&](int, uint32_t k, bool v) {
        g_w += __popc(__ballot_sync(0xffffffffu, v && k > T));
        e_w += __popc(__ballot_sync(0xffffffffu, v && k == T));
    });
    if (lane == 0) {
        s_off[warp][0] = g_w;
        s_off[warp][1] = e_w;
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t g = lane < W ? s_off[lane][0] : 0u, e = lane < W ? s_off[lane][1] : 0u;
        uint32_t gi = g, ei = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t yg = __shfl_up_sync(0xffffffffu, gi, o), ye = __shfl_up_sync(0xffffffffu, ei, o);
            if (lane >= o) {
                gi += yg;
                ei += ye;
            }
        }
        __syncwarp();
        if (lane < W) {
            s_off[lane][0] = gi - g;
            s_off[lane][1] = ei - e;
        }
    }
    __syncthreads();
    uint32_t gb = s_off[warp][0], eb = s_off[warp][1];
    walk([&](int i, uint32_t k, bool v) {
        const bool isg = v && k > T, ise = v && k == T;
        const uint32_t bg = __ballot_sync(0xffffffffu, isg), be = __ballot_sync(0xffffffffu, ise);
        const uint32_t g_before = gb + __popc(bg & lt), e_before = eb + __popc(be & lt);
        if (isg || (ise && e_before < krem)) {
            const uint32_t pos = g_before + (isg ? min(e_before, krem) : e_before);
            if (pos < (uint32_t)kb) out[pos] = i;
            else atomicOr(flag, kFlagBounds);  // unreachable when the select is consistent
        }
        gb += __popc(bg);
        eb += __popc(be);
    });
    for (int p = kb + tid; p < k_max; p += THREADS) out[p] = -1;
}

// Used for many units (at least one per SM) or short units: one CTA each.
bool topk_stream_fits(int units, int rows_cap) { return units >= 148 || rows_cap <= 8192; }

template <int THREADS>
static cudaError_t ts_launch(const float* scores, const int32_t* lens, const int32_t* kreq, int k_max,
                             const Dims& d, int rows_cap, int block, int32_t* idx, uint32_t* hist,
                             unsigned* flag, cudaStream_t st) {
    constexpr int W = THREADS / 32;
    // per-warp list: room for ~4x an even share of k (the boundary bin adds to k)
    int wcap = 64;
    while (wcap < 1024 && (long long)wcap * W < 4LL * k_max) wcap *= 2;
    const size_t smem = (size_t)2 * W * wcap * sizeof(uint32_t);
    static int configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(topk_stream_kernel<THREADS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 2 * W * 1024 * (int)sizeof(uint32_t));
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)d.units());
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, topk_stream_kernel<THREADS>, scores, lens, kreq, k_max, d.Hkv, d.Ncap,
                              rows_cap, block, wcap, idx, hist, flag);
}

cudaError_t launch_topk_stream(const float* scores, const int32_t* lens, const int32_t* kreq, int k_max,
                               const Dims& d, int block, int32_t* idx, uint32_t* hist, unsigned* flag,
                               cudaStream_t st) {
    const int rows_cap = rows_cap_of(d, block);
    // many units: 256 threads (several CTAs per SM); few short units: 512
    const cudaError_t e =
        d.units() >= 148 ? ts_launch<256>(scores, lens, kreq, k_max, d, rows_cap, block, idx, hist, flag, st)
                         : ts_launch<512>(scores, lens, kreq, k_max, d, rows_cap, block, idx, hist, flag, st);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa
