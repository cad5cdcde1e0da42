// topk.cu -- step 2 of the decode path: exact top-k per (sequence, kv-head).
//
// "inference-time context sparsity: illusion or opportunity?", sec. 2: oracle
// Top-K picks exactly the k highest-scoring tokens.  Ties go to the lower
// index and the output is in ascending index order, so the result is unique.
//
// Design (B200): one thread-block cluster of C CTAs per unit (C <= 8, or 16
// when a unit is too long for 8 slices).  Each CTA
// holds its slice of the unit's scores in shared memory as order-preserving
// 32-bit keys, so the scores are read from L2/HBM once.  A radix select with
// 11/11/10-bit digits finds the k-th largest key T exactly:
//   pass 0: every CTA builds a shared-memory histogram of its keys' top digit
//           and adds its non-zero bins into every cluster member's copy of the
//           cluster histogram (remote atomic adds over distributed shared
//           memory); after one cluster barrier each CTA holds the full
//           histogram and finds the bin of T with a block-wide scan from the top
//           (inside a decode step, where the scorer has counted this digit
//           already, topk_hist.cu and topk_stream.cu start from its histogram);
//   filter: one pass over the keys keeps, in index order, those whose top digit
//           is at or above that bin (every selected key plus the candidates of
//           the boundary bin: ~2-10% of the keys);
//   pass 1, 2: on the boundary-bin candidates only: every CTA posts their keys
//           into rank 0's shared memory, rank 0 finishes the select locally and
//           broadcasts T (with the cluster histograms as the fallback when the
//           candidates overflow rank 0's buffer).
// Then keys > T are all taken and keys == T are taken in index order until k
// is reached; positions come from a block scan over the short list and a
// cluster scan of the per-CTA counts.  Cluster barriers are hardware barriers;
// there is no software spin anywhere in this kernel.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace tsa {

constexpr int kTkThreads = 1024;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkLocalPref = 16384;  // keys per CTA before the cluster grows
constexpr int kTkClusterMax = 16;    // 8 (portable) unless a unit needs more shared memory
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
    griddep_wait();
    griddep_launch();

    extern __shared__ __align__(16) uint32_t tk_smem[];
    uint32_t* keys = tk_smem;                                      // [chunk]
    uint32_t* lh = keys + chunk;                                   // [kTkHist] this CTA's histogram
    uint32_t* gh = lh + kTkHist;                                   // [2][kTkHist] cluster histograms
    uint16_t* list = reinterpret_cast<uint16_t*>(gh + 2 * kTkHist);  // [chunk] per-warp filter output
    uint16_t* clist = list + chunk;                                // [chunk] compacted, index order
    uint32_t* cand = reinterpret_cast<uint32_t*>(clist + chunk);   // [chunk/2] rank 0: candidates' keys
    __shared__ uint32_t wsum[33];
    __shared__ uint32_t s_sel[2];
    __shared__ uint32_t s_wcnt[kTkWarps];
    __shared__ uint32_t s_tot[16][2];  // (gt, eq) totals pushed by lower-ranked CTAs
    __shared__ uint32_t s_lc;
    __shared__ uint32_t s_ncand;        // rank 0: candidates received
    __shared__ uint32_t s_Tk[3];        // rank 0 -> all: T, krem, fallback flag

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

    // ---- scores in flight first, then clear the histograms, then one barrier
    const float* su = scores + (size_t)unit * rows_cap + lo;
    constexpr int kBatch = 8;
    float f[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
        const int i = tid + j * kTkThreads;
        f[j] = i < nloc ? __ldcg(su + i) : 0.f;
    }
    // add the non-zero bins into every cluster member's histogram
    auto push_hist = [&](uint32_t* dst_local, int nbins) {
        for (int bin = tid; bin < nbins; bin += kTkThreads) {
            const uint32_t c = lh[bin];
            if (c) {
                for (int r = 0; r < C; ++r) atomicAdd(cluster.map_shared_rank(dst_local + bin, r), c);
            }
        }
    };
    // find, from the top bin down, the bin holding the krem-th largest key
    auto select_bin = [&](const uint32_t* h, int nbins, uint32_t krem) {
        const int hb0 = nbins - 1 - 2 * tid, hb1 = hb0 - 1;
        const uint32_t c0 = hb1 >= 0 ? h[hb0] : 0u, c1 = hb1 >= 0 ? h[hb1] : 0u;
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
    };
    for (int i = tid; i < 3 * kTkHist; i += kTkThreads) lh[i] = 0u;  // lh, gh[0], gh[1]
    if (tid == 0) s_ncand = 0u;
    cluster.sync();  // every CTA's cluster histograms are zero before anyone adds to them

    // ---- pass 0: keys to shared memory, local histogram of the top digit
    for (int i0 = 0; i0 < nloc; i0 += kBatch * kTkThreads) {
        if (i0 > 0) {
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int i = i0 + tid + j * kTkThreads;
                f[j] = i < nloc ? __ldcg(su + i) : 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int i = i0 + tid + j * kTkThreads;
            if (i < nloc) {
                const uint32_t k = order_key(f[j]);
                keys[i] = k;
                atomicAdd(&lh[k >> 21], 1u);
            }
        }
}
    __syncthreads();
    push_hist(gh, kTkHist);
    cluster.sync();  // every CTA now holds the cluster histogram of the top digit
    select_bin(gh, kTkHist, (uint32_t)kb);
    const uint32_t d0 = s_sel[0];
    uint32_t krem = (uint32_t)kb - s_sel[1];

    // ---- filter: keys whose top digit is >= d0, in index order (local indices)
    const int seg = ceil_div(ceil_div(nloc, kTkWarps), 32) * 32;
    const int wbeg = min(warp * seg, nloc), wend = min(wbeg + seg, nloc);
    uint32_t wcnt = 0;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int i0 = wbeg; i0 < wend; i0 += 32) {
        const int i = i0 + lane;
        const bool keep = i < wend && (keys[i] >> 21) >= d0;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) list[wbeg + wcnt + __popc(bal & lt_mask)] = (uint16_t)i;
        wcnt += __popc(bal);
    }
    if (lane == 0) s_wcnt[warp] = wcnt;
    for (int i = tid; i < kTkHist; i += kTkThreads) lh[i] = 0u;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = s_wcnt[lane];
        uint32_t inc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        s_wcnt[lane] = inc - w;  // exclusive offsets
        if (lane == 31) s_lc = inc;
    }
    __syncthreads();
    for (uint32_t j = lane; j < wcnt; j += 32) clist[s_wcnt[warp] + j] = list[wbeg + j];
    __syncthreads();
    const int lc = (int)s_lc;

    // ---- passes 1 and 2 on the boundary-bin candidates.  Only their multiset
    // matters for T, so every CTA posts its candidates' keys into rank 0's
    // shared memory (slots reserved with one remote atomic per CTA); rank 0
    // runs both passes locally and broadcasts (T, krem).  If the candidates do
    // not fit rank 0's buffer (heavy ties), both passes run over the cluster
    // histograms instead.
    const uint32_t cand_cap = (uint32_t)chunk / 2;
    uint32_t nc_local = 0;
    for (int li = tid; li < lc; li += kTkThreads) nc_local += (keys[clist[li]] >> 21) == d0;
    {
        uint32_t tot_c;
        block_excl_scan(nc_local, wsum, &tot_c);
        __shared__ uint32_t s_cbase;
        if (tid == 0) s_cbase = tot_c ? atomicAdd(cluster.map_shared_rank(&s_ncand, 0), tot_c) : 0u;
        __syncthreads();
        const uint32_t cbase = s_cbase;
        // post this CTA's candidates (order free) while there is room
        if (cbase + tot_c <= cand_cap) {
            __shared__ uint32_t s_cpos;
            if (tid == 0) s_cpos = 0;
            __syncthreads();
            uint32_t* dst0 = cluster.map_shared_rank(cand, 0);
            for (int li = tid; li < lc; li += kTkThreads) {
                const uint32_t k = keys[clist[li]];
                if ((k >> 21) == d0) dst0[cbase + atomicAdd(&s_cpos, 1u)] = k;
            }
        }
    }
    cluster.sync();  // every candidate has arrived at rank 0 (or rank 0 knows it overflowed)
    if (rank == 0) {
        const uint32_t nc = s_ncand;
        const bool fits = nc <= cand_cap;
        uint32_t pre = d0 << 21, pm = 0x7ffu << 21, kr = krem;
        if (fits) {
#pragma unroll 1
            for (int p = 1; p < 3; ++p) {
                const int shift = p == 1 ? 10 : 0;
                const int nbins = p == 1 ? 2048 : 1024;
                const uint32_t dmask = (uint32_t)nbins - 1u;
                for (int i = tid; i < kTkHist; i += kTkThreads) lh[i] = 0u;
                __syncthreads();
                for (uint32_t i = tid; i < nc; i += kTkThreads) {
                    const uint32_t k = cand[i];
                    if ((k & pm) == pre) atomicAdd(&lh[(k >> shift) & dmask], 1u);
                }
                __syncthreads();
                select_bin(lh, nbins, kr);
                pre |= s_sel[0] << shift;
                pm |= dmask << shift;
                kr -= s_sel[1];
                __syncthreads();
            }
        }
        if (tid < C) {
            uint32_t* d = cluster.map_shared_rank(s_Tk, tid);
            d[0] = pre;
            d[1] = kr;
            d[2] = fits ? 0u : 1u;
        }
    }
    cluster.sync();  // (T, krem) or the fallback flag is everywhere
    uint32_t prefix = s_Tk[0];
    if (s_Tk[2]) {  // fallback: passes 1 and 2 over the cluster histograms
        prefix = d0 << 21;
        uint32_t pmask = 0x7ffu << 21;
        for (int i = tid; i < kTkHist; i += kTkThreads) lh[i] = 0u;
        __syncthreads();
#pragma unroll 1
        for (int p = 1; p < 3; ++p) {
            const int shift = p == 1 ? 10 : 0;
            const int nbins = p == 1 ? 2048 : 1024;
            const uint32_t dmask = (uint32_t)nbins - 1u;
            uint32_t* g = gh + (p & 1) * kTkHist;
            for (int li = tid; li < lc; li += kTkThreads) {
                const uint32_t k = keys[clist[li]];
                if ((k & pmask) == prefix) atomicAdd(&lh[(k >> shift) & dmask], 1u);
            }
            // the other cluster histogram is free again (read before the last barrier): clear it
            uint32_t* other = gh + ((p + 1) & 1) * kTkHist;
            for (int i = tid; i < kTkHist; i += kTkThreads) other[i] = 0u;
            __syncthreads();
            push_hist(g, nbins);
            for (int i = tid; i < kTkHist; i += kTkThreads) lh[i] = 0u;
            cluster.sync();
            select_bin(g, nbins, krem);
            prefix |= s_sel[0] << shift;
            pmask |= dmask << shift;
            krem -= s_sel[1];
            __syncthreads();
        }
    } else {
        krem = s_Tk[1];
    }
    const uint32_t T = prefix;  // the k-th largest key; krem keys equal to T are taken

    // ---- positions: block scan of (> T, == T) over the list, cluster scan of CTA totals
    const int per = ceil_div(lc, kTkThreads);
    const int beg = min(tid * per, lc), end = min(beg + per, lc);
    uint32_t ng = 0, ne = 0;
    for (int li = beg; li < end; ++li) {
        const uint32_t k = keys[clist[li]];
        ng += k > T;
        ne += k == T;
    }
    uint32_t tot;
    const uint32_t ex = block_excl_scan((ng << 16) | ne, wsum, &tot);  // lc <= chunk < 65536
    if (tid < C && tid > rank) {  // push this CTA's totals to every higher-ranked CTA
        uint32_t* dst = cluster.map_shared_rank(&s_tot[rank][0], tid);
        dst[0] = tot >> 16;
        dst[1] = tot & 0xffffu;
    }
    cluster.sync();  // totals of all lower ranks have arrived
    uint32_t gb = ex >> 16, eb = ex & 0xffffu;
    for (int r = 0; r < rank; ++r) {
        gb += s_tot[r][0];
        eb += s_tot[r][1];
    }
    for (int li = beg; li < end; ++li) {
        const int i = clist[li];
        const uint32_t k = keys[i];
        const bool isg = k > T, ise = k == T;
        if (isg || (ise && eb < krem)) {
            const uint32_t pos = isg ? gb + min(eb, krem) : gb + eb;
            if (pos < (uint32_t)kb) out[pos] = lo + i;
            else atomicOr(flag, kFlagBounds);  // unreachable when the select is consistent
        }
        gb += isg;
        eb += ise;
    }
    if (rank == 0)
        for (int p = kb + tid; p < k_max; p += kTkThreads) out[p] = -1;
    // no distributed-shared-memory access follows the last barrier
}

static size_t topk_smem_bytes(int chunk) {
    // keys, lh + gh[2], two u16 lists, rank 0's candidate buffer (chunk/2 keys)
    return (size_t)chunk * 4 + 3 * kTkHist * 4 + (size_t)chunk * 2 * 2 + (size_t)(chunk / 2) * 4;
}

bool topk_plan(int rows_cap, int* cluster, int* chunk) {
    int C = 1;  // grow to 8 by the preferred slice size, to 16 only when 8 slices do not fit
    while (C < 8 && ceil_div(rows_cap, C) > kTkLocalPref) C *= 2;
    if (topk_smem_bytes(ceil_div(ceil_div(rows_cap, C), 32) * 32) > 200 * 1024) C = kTkClusterMax;
    int ch = ceil_div(rows_cap, C);
    ch = ceil_div(ch, 32) * 32;
    if (ch < 32) ch = 32;
    if (topk_smem_bytes(ch) > 200 * 1024) return false;
    *cluster = C;
    *chunk = ch;
    return true;
}

static int g_tk_configured[64];

cudaError_t launch_topk(const float* scores, const int32_t* lens, const int32_t* kreq, int k_max,
                        const Dims& d, int block, int32_t* idx, uint32_t* hist, unsigned* flag,
                        cudaStream_t st) {
    if (d.units() == 0 || k_max == 0) return cudaSuccess;
    const int rows_cap = rows_cap_of(d, block);
    if (topk_stream_fits(d.units(), rows_cap))
        return launch_topk_stream(scores, lens, kreq, k_max, d, block, idx, hist, flag, st);
    int hc = 1, hk = 16;
    if (hist && topk_hist_plan(d.units(), rows_cap, &hc, &hk))
        return launch_topk_hist(hc, hk, scores, lens, kreq, k_max, d, block, idx, hist, flag, st);
    if (hist) {  // a shape neither histogram-fed kernel takes: count afresh, leave the counts zero
        const cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)d.units() * kHistBins * sizeof(uint32_t), st);
        if (e != cudaSuccess) return e;
    }
    int C = 1, chunk = 32;
    if (!topk_plan(rows_cap, &C, &chunk)) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !g_tk_configured[dev]) {
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        g_tk_configured[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(d.units() * C));
    cfg.blockDim = dim3(kTkThreads);
    cfg.dynamicSmemBytes = topk_smem_bytes(chunk);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, topk_kernel, scores, lens, kreq, k_max, d.Hkv, d.Ncap, rows_cap,
                           block, chunk, idx, flag);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa
