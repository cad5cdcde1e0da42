// topk_hist.cu -- step 2 of the decode path inside a decode step, for few long
// units: exact top-k per (sequence, kv-head), starting from the scorer's
// histogram of the first radix digit.
//
// "inference-time context sparsity: illusion or opportunity?", sec. 2: oracle
// Top-K picks exactly the k highest-scoring tokens.  Ties go to the lower
// index and the output is in ascending index order, so the result is unique.
//
// The scorer of the same step has counted the top 11 bits of every score key
// (its epilogue, hidden behind HBM).  So the bin d0 of the k-th largest key is
// known before any score is looked at, and the kernel's critical path is short:
//   1. each CTA of the unit's cluster (C CTAs x 1024 threads, KPT scores a
//      thread) issues its score loads, copies the histogram and finds d0 while
//      they are in flight;
//   2. the loaded scores are filtered in registers (a batch of raw floats
//      against d0's smallest float first, then the exact key test) into
//      per-warp lists in shared memory: warp w owns a contiguous run of rows,
//      so the lists are in index order with no sort;
//   3. the keys of bin d0 are posted into rank 0's shared memory (one remote
//      atomic per warp reserves the slots); rank 0 resolves the next 11 bits
//      over them, the last 10 over the few keys left, and broadcasts T (the
//      k-th largest key) and krem (how many keys equal to T to take);
//   4. keys > T and the first krem keys == T get their output positions from a
//      count per warp, a scan over the warps and a cluster scan of the CTAs.
// Three cluster barriers in all; no software spin.  When a list or rank 0's
// buffer would overflow (heavy ties, k near the length), steps 3 and 4 run
// over every register-held key instead, with the digits resolved over cluster
// histograms.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace tsa {

constexpr int kThThreads = 1024;
constexpr int kThWarps = 32;
constexpr int kThWcap = 128;                   // list entries per warp
constexpr int kThCandCap = 8192;               // rank 0's buffer for bin d0's keys
constexpr int kThClusterMax = 16;

struct ThSmem {
    uint32_t gh[kHistBins];                    // the unit's digit-1 histogram, then cluster histograms (fallback)
    uint32_t ph[kHistBins];                    // rank 0: digit-2 and digit-3 histograms; fallback: local
    uint32_t lkey[kThWarps * kThWcap];         // per-warp lists: keys ...
    uint32_t lrow[kThWarps * kThWcap];         // ... and their rows (CTA-local)
    uint32_t cand[kThCandCap];                 // rank 0: bin d0's keys
    uint32_t wsum[33];
    uint32_t wcnt[kThWarps];                   // entries per warp list
    uint32_t wge[kThWarps][2];                 // per-warp (gt, eq) counts, then offsets
    uint32_t tot[kThClusterMax][2];            // (gt, eq) totals pushed by lower-ranked CTAs
    uint32_t sel[2];
    uint32_t ncand;                            // rank 0: keys posted
    uint32_t over;                             // rank 0: some list overflowed
    uint32_t Tk[3];                            // rank 0 -> all: T, krem, fallback
    uint32_t small[64];                        // rank 0: keys sharing the first two digits
    uint32_t nsmall;
};

__device__ __forceinline__ uint32_t th_block_scan(uint32_t x, uint32_t* wsum, uint32_t* total) {
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

template <int KPT>
__global__ void __launch_bounds__(kThThreads, 1)
topk_hist_kernel(const float* __restrict__ scores, const int32_t* __restrict__ lens,
                 const int32_t* __restrict__ kreq, int k_max, int Hkv, int Ncap, int rows_cap, int block,
                 int32_t* __restrict__ idx, uint32_t* __restrict__ hist, unsigned* __restrict__ flag) {
    constexpr int kSeg = 32 * KPT;             // a warp's run of rows
    constexpr int kChunk = kThWarps * kSeg;    // a CTA's rows
    extern __shared__ __align__(16) unsigned char th_raw[];
    ThSmem& sm = *reinterpret_cast<ThSmem*>(th_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int unit = blockIdx.x / C;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    // the lengths and k's are not the scorer's output: read them before waiting on it
    int len = lens[b];
    int kb = kreq ? kreq[b] : k_max;
    griddep_wait();
    griddep_launch();

    // ---- 1. score loads and the histogram copy go out first (the scores
    // buffer holds rows_cap rows a unit, so the slice is in bounds whatever
    // len_b is; rows past len_b are masked below), then the lengths
    const int lo = rank * kChunk;
    const int wbase = warp * kSeg;
    const int lim = min(kChunk, rows_cap - lo);
    const float* su = scores + (size_t)unit * rows_cap + lo;
    uint32_t* hu = hist + (size_t)unit * kHistBins;
    float f[KPT];
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int i = wbase + j * 32 + lane;
        f[j] = i < lim ? __ldcg(su + i) : 0.f;
    }
    if (tid < kHistBins / 4) reinterpret_cast<uint4*>(sm.gh)[tid] = __ldcg(reinterpret_cast<const uint4*>(hu) + tid);

    if (len < 0 || len > Ncap) {
        if (tid == 0 && rank == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    const int n = block == 1 ? len : ceil_div(len, block);
    if (kb < 0) kb = 0;
    if (kb > n) kb = n;
    if (kb > k_max) {
        if (tid == 0 && rank == 0) atomicOr(flag, kFlagBounds);
        kb = k_max;
    }
    int32_t* out = idx + (size_t)unit * k_max;
    const int nloc = max(0, min(kChunk, n - lo));

    // Degenerate units need no selection; every CTA of the cluster takes the
    // same branch, so no cluster barrier is left waiting.
    if (kb == 0 || kb == n) {
        for (int i = tid; i < nloc; i += kThThreads)
            if (lo + i < kb) out[lo + i] = lo + i;
        if (rank == 0) {
            for (int p = kb + tid; p < k_max; p += kThThreads) out[p] = -1;
            for (int i = tid; i < kHistBins; i += kThThreads) hu[i] = 0u;  // ready for the next step
        }
        return;
    }

    // ---- d0 while the scores land
    for (int i = tid; i < kHistBins; i += kThThreads) sm.ph[i] = 0u;
    if (tid == 0) {
        sm.ncand = 0u;
        sm.over = 0u;
    }
    // split cluster barrier: arrive once the copy is taken and the counters are
    // zero; wait before the first remote access (and before rank 0 zeroes hu)
    asm volatile("barrier.cluster.arrive.aligned;\n" ::: "memory");
    __syncthreads();

    // from the top bin down, the bin holding the kr-th largest key (2 bins a thread)
    auto select_bin = [&](const uint32_t* h, int nbins, uint32_t kr) {
        const int hb0 = nbins - 1 - 2 * tid, hb1 = hb0 - 1;
        const uint32_t c0 = hb1 >= 0 ? h[hb0] : 0u, c1 = hb1 >= 0 ? h[hb1] : 0u;
        uint32_t total;
        const uint32_t above = th_block_scan(c0 + c1, sm.wsum, &total);
        if (hb1 >= 0 && above < kr && kr <= above + c0 + c1) {  // exactly one thread
            if (kr <= above + c0) {
                sm.sel[0] = (uint32_t)hb0;
                sm.sel[1] = above;
            } else {
                sm.sel[0] = (uint32_t)hb1;
                sm.sel[1] = above + c0;
            }
        }
        __syncthreads();
    };
    select_bin(sm.gh, kHistBins, (uint32_t)kb);
    const uint32_t d0 = sm.sel[0];
    uint32_t krem = (uint32_t)kb - sm.sel[1];

    // ---- 2. filter the registers into this warp's list (index order)
    uint32_t* lkey = sm.lkey + warp * kThWcap;
    uint32_t* lrow = sm.lrow + warp * kThWcap;
    uint32_t cnt = 0;  // list entries
    {
        const uint32_t kthr = d0 << 21;
        const float fthr = __uint_as_float((kthr & 0x80000000u) ? (kthr & 0x7fffffffu) : ~kthr);
        bool any = false;
#pragma unroll
        for (int j = 0; j < KPT; ++j) any |= (wbase + j * 32 + lane < nloc) && !(f[j] < fthr);
        if (__any_sync(0xffffffffu, any)) {
#pragma unroll
            for (int j = 0; j < KPT; ++j) {
                const int i = wbase + j * 32 + lane;
                const uint32_t k = order_key(f[j]);
                const bool keep = i < nloc && (k >> 21) >= d0;
                const uint32_t bal = __ballot_sync(0xffffffffu, keep);
                const uint32_t pos = cnt + __popc(bal & lt);
                if (keep && pos < (uint32_t)kThWcap) {
                    lkey[pos] = k;
                    lrow[pos] = (uint32_t)i;
                }
                cnt += __popc(bal);
            }
        }
    }
    for (int i = tid; i < kHistBins; i += kThThreads) sm.gh[i] = 0u;  // rank 0's digit-3 histogram, zero early
    asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory");
    if (rank == 0)
        for (int i = tid; i < kHistBins; i += kThThreads) hu[i] = 0u;  // every member has its copy
    // ---- 3. bin d0's keys to rank 0 (a warp reserves its slots with one remote
    // atomic), and their second digit into rank 0's histogram on the way
    const bool wover = cnt > (uint32_t)kThWcap;
    if (lane == 0) {
        sm.wcnt[warp] = cnt;
        if (wover) atomicOr(cluster.map_shared_rank(&sm.over, 0), 1u);
    }
    if (!wover) {
        uint32_t ncw = 0;
        for (uint32_t e0 = 0; e0 < cnt; e0 += 32) {
            const uint32_t e = e0 + lane;
            ncw += __popc(__ballot_sync(0xffffffffu, e < cnt && (lkey[e] >> 21) == d0));
        }
        uint32_t base = 0;
        if (lane == 0 && ncw) base = atomicAdd(cluster.map_shared_rank(&sm.ncand, 0), ncw);
        base = __shfl_sync(0xffffffffu, base, 0);
        if (ncw && base + ncw <= (uint32_t)kThCandCap) {
            uint32_t* dst = cluster.map_shared_rank(sm.cand, 0) + base;
            uint32_t off = 0;
            for (uint32_t e0 = 0; e0 < cnt; e0 += 32) {
                const uint32_t e = e0 + lane;
                const uint32_t k = e < cnt ? lkey[e] : 0u;
                const bool c = e < cnt && (k >> 21) == d0;
                const uint32_t bal = __ballot_sync(0xffffffffu, c);
                if (c) dst[off + __popc(bal & lt)] = k;
                off += __popc(bal);
            }
        }
    }
    cluster.sync();  // bin d0's keys are at rank 0 (or it knows of an overflow)

    if (rank == 0) {
        const uint32_t nc = sm.ncand;
        const bool fits = nc <= (uint32_t)kThCandCap && sm.over == 0u;
        uint32_t pre = d0 << 21, pm = 0x7ffu << 21, kr = krem;
        if (fits) {
            // digit 2 over bin d0's keys (local atomics: ~4 a thread)
            for (uint32_t i = tid; i < nc; i += kThThreads) atomicAdd(&sm.ph[(sm.cand[i] >> 10) & 0x7ffu], 1u);
            __syncthreads();
            select_bin(sm.ph, 2048, kr);
            pre |= sm.sel[0] << 10;
            pm |= 0x7ffu << 10;
            kr -= sm.sel[1];
            // digit 3: the keys sharing the first two are usually a handful, so
            // one warp ranks them directly; more (ties) take a histogram pass
            if (tid == 0) sm.nsmall = 0u;
            __syncthreads();
            for (uint32_t i = tid; i < nc; i += kThThreads) {
                const uint32_t k = sm.cand[i];
                if ((k & pm) == pre) {
                    const uint32_t q = atomicAdd(&sm.nsmall, 1u);
                    if (q < 64u) sm.small[q] = k;
                }
            }
            __syncthreads();
            const uint32_t ns = sm.nsmall;  // >= kr >= 1
            if (ns <= 64u) {
                if (warp == 0) {
                    // T is the key x with #{y > x} < kr <= #{y >= x}; krem = kr - #{y > x}
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t me = (uint32_t)(lane + 32 * h);
                        if (me < ns) {
                            const uint32_t x = sm.small[me];
                            uint32_t gt = 0, ge = 0;
                            for (uint32_t j = 0; j < ns; ++j) {
                                const uint32_t y = sm.small[j];
                                gt += y > x;
                                ge += y >= x;
                            }
                            if (gt < kr && kr <= ge) {  // every lane holding T writes the same
                                sm.sel[0] = x;
                                sm.sel[1] = gt;
                            }
                        }
                    }
                }
                __syncthreads();
                pre = sm.sel[0];
                kr -= sm.sel[1];
            } else {
                for (uint32_t i = tid; i < nc; i += kThThreads) {
                    const uint32_t k = sm.cand[i];
                    if ((k & pm) == pre) atomicAdd(&sm.gh[k & 0x3ffu], 1u);
                }
                __syncthreads();
                select_bin(sm.gh, 1024, kr);
                pre |= sm.sel[0];
                kr -= sm.sel[1];
            }
        }
        if (tid < C) {
            uint32_t* d = cluster.map_shared_rank(sm.Tk, tid);
            d[0] = pre;
            d[1] = kr;
            d[2] = fits ? 0u : 1u;
        }
    }
    cluster.sync();  // (T, krem) or the fallback flag is everywhere
    const bool fallback = sm.Tk[2] != 0u;
    uint32_t T = sm.Tk[0];
    if (fallback) {
        // digits 2 and 3 over cluster histograms of every register-held key
        uint32_t prefix = d0 << 21, pmask = 0x7ffu << 21;
#pragma unroll 1
        for (int p = 1; p < 3; ++p) {
            const int shift = p == 1 ? 10 : 0;
            const int nbins = p == 1 ? 2048 : 1024;
            const uint32_t dmask = (uint32_t)nbins - 1u;
            for (int i = tid; i < kHistBins; i += kThThreads) {
                sm.gh[i] = 0u;
                sm.ph[i] = 0u;
            }
            cluster.sync();  // zero everywhere (and every earlier read of gh done)
#pragma unroll
            for (int j = 0; j < KPT; ++j) {
                const uint32_t k = order_key(f[j]);
                if (wbase + j * 32 + lane < nloc && (k & pmask) == prefix) atomicAdd(&sm.ph[(k >> shift) & dmask], 1u);
            }
            __syncthreads();
            for (int bin = tid; bin < nbins; bin += kThThreads) {
                const uint32_t c = sm.ph[bin];
                if (c)
                    for (int r = 0; r < C; ++r) atomicAdd(cluster.map_shared_rank(&sm.gh[bin], r), c);
            }
            cluster.sync();
            select_bin(sm.gh, nbins, krem);
            prefix |= sm.sel[0] << shift;
            pmask |= dmask << shift;
            krem -= sm.sel[1];
        }
        T = prefix;
    } else {
        krem = sm.Tk[1];
    }

    // ---- 4. output: keys > T, and keys == T in index order while fewer than krem
    // f(row, key, valid) over this warp's keys still in play, in index order
    auto walk = [&](auto&& fn) {
        if (!fallback) {
            for (uint32_t e0 = 0; e0 < cnt; e0 += 32) {
                const uint32_t e = e0 + lane;
                const bool v = e < cnt;
                fn(v ? (int)lrow[e] : 0, v ? lkey[e] : 0u, v);
            }
        } else {
#pragma unroll
            for (int j = 0; j < KPT; ++j) {
                const int i = wbase + j * 32 + lane;
                fn(i, order_key(f[j]), i < nloc);
            }
        }
    };
    uint32_t g_w = 0, e_w = 0;
    walk([&](int, uint32_t k, bool v) {
        g_w += __popc(__ballot_sync(0xffffffffu, v && k > T));
        e_w += __popc(__ballot_sync(0xffffffffu, v && k == T));
    });
    if (lane == 0) {
        sm.wge[warp][0] = g_w;
        sm.wge[warp][1] = e_w;
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the warps' counts; CTA totals to every higher rank
        const uint32_t g = sm.wge[lane][0], e = sm.wge[lane][1];
        uint32_t gi = g, ei = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t yg = __shfl_up_sync(0xffffffffu, gi, o), ye = __shfl_up_sync(0xffffffffu, ei, o);
            if (lane >= o) {
                gi += yg;
                ei += ye;
            }
        }
        sm.wge[lane][0] = gi - g;
        sm.wge[lane][1] = ei - e;
        const uint32_t gt = __shfl_sync(0xffffffffu, gi, 31), et = __shfl_sync(0xffffffffu, ei, 31);
        if (lane > rank && lane < C) {
            uint32_t* dst = cluster.map_shared_rank(&sm.tot[rank][0], lane);
            dst[0] = gt;
            dst[1] = et;
        }
    }
    cluster.sync();  // totals of all lower ranks have arrived
    uint32_t gb = sm.wge[warp][0], eb = sm.wge[warp][1];
    for (int r = 0; r < rank; ++r) {
        gb += sm.tot[r][0];
        eb += sm.tot[r][1];
    }
    walk([&](int i, uint32_t k, bool v) {
        const bool isg = v && k > T, ise = v && k == T;
        const uint32_t bg = __ballot_sync(0xffffffffu, isg), be = __ballot_sync(0xffffffffu, ise);
        const uint32_t g_before = gb + __popc(bg & lt), e_before = eb + __popc(be & lt);
        if (isg || (ise && e_before < krem)) {
            const uint32_t pos = g_before + (isg ? min(e_before, krem) : e_before);
            if (pos < (uint32_t)kb) out[pos] = lo + i;
            else atomicOr(flag, kFlagBounds);  // unreachable when the select is consistent
        }
        gb += __popc(bg);
        eb += __popc(be);
    });
    if (rank == 0)
        for (int p = kb + tid; p < k_max; p += kThThreads) out[p] = -1;
    // no distributed-shared-memory access follows the last barrier
}

// Used inside a decode step (the scorer's histogram is there) for few long
// units; keys a thread 16 (32 past 8 x 16384 rows), clusters of up to 16.
bool topk_hist_plan(int units, int rows_cap, int* cluster, int* kpt) {
    if (topk_stream_fits(units, rows_cap)) return false;
    int k = 16, C = ceil_div(rows_cap, kThThreads * k);
    if (C > 8) {
        k = 32;
        C = ceil_div(rows_cap, kThThreads * k);
    }
    if (C > kThClusterMax) return false;
    *cluster = C;
    *kpt = k;
    return true;
}

template <int KPT>
static cudaError_t th_launch(int C, const float* scores, const int32_t* lens, const int32_t* kreq, int k_max,
                             const Dims& d, int rows_cap, int block, int32_t* idx, uint32_t* hist,
                             unsigned* flag, cudaStream_t st) {
    static int configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(topk_hist_kernel<KPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(ThSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(topk_hist_kernel<KPT>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(d.units() * C));
    cfg.blockDim = dim3(kThThreads);
    cfg.dynamicSmemBytes = sizeof(ThSmem);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, topk_hist_kernel<KPT>, scores, lens, kreq, k_max, d.Hkv, d.Ncap, rows_cap,
                              block, idx, hist, flag);
}

cudaError_t launch_topk_hist(int C, int kpt, const float* scores, const int32_t* lens, const int32_t* kreq,
                             int k_max, const Dims& d, int block, int32_t* idx, uint32_t* hist, unsigned* flag,
                             cudaStream_t st) {
    const int rows_cap = rows_cap_of(d, block);
    const cudaError_t e =
        kpt == 16 ? th_launch<16>(C, scores, lens, kreq, k_max, d, rows_cap, block, idx, hist, flag, st)
                  : th_launch<32>(C, scores, lens, kreq, k_max, d, rows_cap, block, idx, hist, flag, st);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa
