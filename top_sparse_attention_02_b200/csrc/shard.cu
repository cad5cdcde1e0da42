// shard.cu -- sequence-sharded decode: one sequence's cache split by rows across
// R ranks, with one exchange of top-k candidates and one of attention partials.
//
// Shard r holds the cache rows [row0_r, row0_r + Ncap_r) of every (b, kv-head)
// unit, row0 increasing with r.  The exact global top-k is found from the
// shards' own top-k lists: every row of the global top-k is among the k largest
// of its shard (fewer than k rows of the shard outrank it), so the global top-k
// of the union of the shards' lists is the global top-k of the cache, and with
// the shards concatenated in row order the lower-index tie rule is kept.  The
// attention splits the same way flash decoding splits a sequence: each shard
// attends over the selected rows it holds and returns its normalised output
// with the base-2 log-sum-exp of its logits, and the parts combine exactly.
//
// Kernels (all small next to the scorer's pass over K):
//   shard_pack     after the shard's top-k: candidate scores and global rows;
//   merge_topk     the exact top-k of a unit's candidates from all R shards in
//                  one CTA (when they fit its shared memory), else:
//   merge_pack     the R shards' candidates of a unit, compacted in row order;
//   merge_map      positions chosen by the top-k over them -> global rows;
//   localize       the global list -> this shard's local rows, at the front;
//   shard_combine  O = sum_r 2^(lse_r - M) O_r / sum_r 2^(lse_r - M).
#include <cmath>

#include "common.cuh"

namespace tsa {

namespace {

constexpr int kShThreads = 256;

// Every glue kernel runs one element a thread over a (chunks, units) grid: the
// lists are a few thousand entries a unit, so the time is the latency of one or
// two loads, not a loop of them.  Counts a chunk needs from the whole list (a
// shard's candidates, the rows below row0) are recomputed by every chunk's CTA
// from independent loads.

// block-wide sum (all threads get it); uses s[0..32]
__device__ __forceinline__ int sh_block_sum(int x, int* s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    __syncthreads();  // s is free (a previous sum has been read)
    if (lane == 0) s[warp] = x;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += s[w];
    return t;
}

// block-wide minimum (all threads get it); uses s[0..32]
__device__ __forceinline__ int sh_block_min(int x, int* s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
    __syncthreads();
    if (lane == 0) s[warp] = x;
    __syncthreads();
    int t = s[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) t = min(t, s[w]);
    return t;
}

__global__ void __launch_bounds__(kShThreads) shard_pack_kernel(const float* __restrict__ scores, int rows_cap,
                                                               int32_t* __restrict__ cand_rows,
                                                               float* __restrict__ cand_scores, int k_max,
                                                               int row0, unsigned* flag) {
    const int u = blockIdx.y, t = blockIdx.x * kShThreads + threadIdx.x;
    if (t >= k_max) return;
    const size_t o = (size_t)u * k_max + t;
    const int r = cand_rows[o];
    if (r >= 0 && r < rows_cap) {
        cand_scores[o] = scores[(size_t)u * rows_cap + r];
        cand_rows[o] = row0 + r;
    } else {
        if (r >= rows_cap) atomicOr(flag, kFlagBounds);
        cand_scores[o] = -INFINITY;
        cand_rows[o] = -1;
    }
}

// the R shards' candidates of a unit (each list: valid rows, then -1) packed
// one after another, then padded with (-inf, -1); CTA x writes packed
// positions [x*256, x*256 + 256), and counts their scores' first radix digit
// into the unit's histogram for the top-k over them
__global__ void __launch_bounds__(kShThreads) merge_pack_kernel(const float* __restrict__ cand_scores,
                                                               const int32_t* __restrict__ cand_rows, int R,
                                                               int units, int Hkv, int k_max,
                                                               float* __restrict__ pk_scores,
                                                               int32_t* __restrict__ pk_rows,
                                                               int32_t* __restrict__ n_cand, uint32_t* __restrict__ hist,
                                                               unsigned* flag) {
    __shared__ int s_off[kMaxShards + 1];
    __shared__ int s_red[33];
    const int u = blockIdx.y, tid = threadIdx.x;
    const int width = R * k_max;
    // each shard's count: the entries before its first -1
    for (int r = 0; r < R; ++r) {
        const int32_t* cr = cand_rows + ((size_t)r * units + u) * k_max;
        int c = k_max;
        for (int t = tid; t < k_max; t += kShThreads)
            if (cr[t] < 0) {
                c = t;
                break;
            }
        c = sh_block_min(c, s_red);
        if (tid == 0) s_off[r] = c;
    }
    __syncthreads();
    if (tid == 0) {  // counts -> offsets; the shards must come in row order (checked once a unit)
        int off = 0, last = -1;
        for (int r = 0; r < R; ++r) {
            const int c = s_off[r];
            if (blockIdx.x == 0 && c > 0) {
                const int32_t* cr = cand_rows + ((size_t)r * units + u) * k_max;
                if (cr[0] <= last) atomicOr(flag, kFlagBounds);
                last = cr[c - 1];
            }
            s_off[r] = off;
            off += c;
        }
        s_off[R] = off;
        if (blockIdx.x == 0 && u % Hkv == 0) n_cand[u / Hkv] = off;  // the same for every kv-head of a sequence
    }
    __syncthreads();
    const int p = blockIdx.x * kShThreads + tid;
    if (p >= width) return;
    float* ps = pk_scores + (size_t)u * width;
    int32_t* pr = pk_rows + (size_t)u * width;
    if (p >= s_off[R]) {
        ps[p] = -INFINITY;
        pr[p] = -1;
        return;
    }
    int r = 0;
    while (s_off[r + 1] <= p) ++r;  // the shard of packed position p
    const size_t src = ((size_t)r * units + u) * k_max + (p - s_off[r]);
    const float sc = cand_scores[src];
    ps[p] = sc;
    pr[p] = cand_rows[src];
    atomicAdd(&hist[(size_t)u * kHistBins + (order_key(sc) >> 21)], 1u);
}

// ---- the merge in one kernel: one CTA (1024 threads) per unit
//
// The R shards' lists stay where they are, [shard][k_max] in shared memory as
// (order key, global row); an entry counts when it lies before its shard's
// first -1.  With the shards in row order, those entries in that order are the
// union in ascending row order, so "first in order" is "lowest row" (the tie
// rule) and no packing is needed.  Three radix passes of shared-memory
// histograms (11, 11 and 10 bits) find T, the k-th largest key, and krem, how
// many keys equal to T to take; block scans over each thread's contiguous run
// of entries give every chosen row its output position.  Replaces pack ->
// top-k -> map (three launches and two trips through the workspace).
// exclusive scan over a block of W warps (all threads get their prefix and the total)
template <int W>
__device__ __forceinline__ uint32_t mg_block_scan(uint32_t x, uint32_t* ws, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) ws[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = lane < W ? ws[lane] : 0u;
        uint32_t winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += y;
        }
        if (lane < W) ws[lane] = winc - w;
        if (lane == 31) ws[32] = winc;
    }
    __syncthreads();
    const uint32_t ex = ws[warp] + inc - x;
    *total = ws[32];
    __syncthreads();  // ws is free for the next scan
    return ex;
}

// A unit is one CTA: its instructions, issued by THREADS / 128 warps a
// sub-partition, are the cost, so every per-entry step is a few instructions
// (no division: an entry past its shard's first -1 is marked by row -1 once).
template <int THREADS>
__global__ void __launch_bounds__(THREADS) merge_topk_kernel(const float* __restrict__ cand_scores,
                                                            const int32_t* __restrict__ cand_rows, int R,
                                                            int units, int Hkv, int k_max,
                                                            const int32_t* __restrict__ kreq,
                                                            int32_t* __restrict__ idx, unsigned* flag) {
    constexpr int W = THREADS / 32;
    extern __shared__ __align__(16) uint32_t mg_smem[];
    __shared__ uint32_t hist[kHistBins];
    __shared__ int s_first[kMaxShards];  // each shard's first -1 (its count)
    __shared__ uint32_t s_ws[33];
    __shared__ uint32_t s_sel[2];        // a pass's bin and the keys above it
    const int u = blockIdx.x, b = u / Hkv, tid = threadIdx.x;
    const int width = R * k_max;
    uint32_t* skey = mg_smem;
    int32_t* srow = reinterpret_cast<int32_t*>(mg_smem + width);
    for (int r = tid; r < R; r += THREADS) s_first[r] = k_max;
    __syncthreads();
    // every shard's list, four entries a thread in flight at a time
    for (int r = 0; r < R; ++r) {
        const int32_t* crr = cand_rows + ((size_t)r * units + u) * k_max;
        const float* csr = cand_scores + ((size_t)r * units + u) * k_max;
        for (int i0 = 0; i0 < k_max; i0 += 4 * THREADS) {
            int32_t rv[4];
            float sv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * THREADS + tid;
                rv[j] = i < k_max ? crr[i] : -1;
                sv[j] = i < k_max ? csr[i] : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * THREADS + tid;
                if (i < k_max) {
                    srow[r * k_max + i] = rv[j];
                    skey[r * k_max + i] = order_key(sv[j]);
                    if (rv[j] < 0) atomicMin(&s_first[r], i);
                }
            }
        }
    }
    __syncthreads();
    // entries past a shard's first -1 are not candidates, whatever they hold
    int n = 0;
    for (int r = 0; r < R; ++r) {
        const int c = s_first[r];
        n += c;
        for (int i = c + tid; i < k_max; i += THREADS) srow[r * k_max + i] = -1;
    }
    if (tid == 0) {  // the shards must come in row order
        int last = -1;
        for (int r = 0; r < R; ++r) {
            const int c = s_first[r];
            if (c == 0) continue;
            if (srow[r * k_max] <= last) atomicOr(flag, kFlagBounds);
            last = srow[r * k_max + c - 1];
        }
    }
    __syncthreads();
    int kb = kreq ? kreq[b] : k_max;
    if (kb < 0) kb = 0;
    if (kb > n) kb = n;
    if (kb > k_max) {
        if (tid == 0) atomicOr(flag, kFlagBounds);
        kb = k_max;
    }
    int32_t* out = idx + (size_t)u * k_max;
    // each thread's contiguous run of entries, for the output in row order
    const int cpt = ceil_div(width, THREADS);
    const int lo = min(width, tid * cpt), hi = min(width, lo + cpt);
    uint32_t T = 0, krem = 0;
    if (kb > 0 && kb < n) {
        // The candidates are all near the top of their shards, so their keys
        // share the high bits (sign, most of the exponent): the digits start
        // below the highest bit in which two keys differ (11 bits a pass, at
        // most 3), so that the first pass spreads them over many bins.
        uint32_t kmin = 0xffffffffu, kmax = 0u;
        for (int t = tid; t < width; t += THREADS)
            if (srow[t] >= 0) {
                kmin = min(kmin, skey[t]);
                kmax = max(kmax, skey[t]);
            }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        }
        if ((tid & 31) == 0) {
            s_ws[tid >> 5] = kmin;
            hist[tid >> 5] = kmax;  // hist is free until the first pass
        }
        __syncthreads();
        kmin = (tid & 31) < W ? s_ws[tid & 31] : 0xffffffffu;
        kmax = (tid & 31) < W ? hist[tid & 31] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        }
        __syncthreads();  // s_ws and hist are free again
        const uint32_t diff = kmin ^ kmax;
        int top_bit = diff ? 31 - __clz(diff) : -1;  // every valid key equal: no pass
        // the bits above top_bit (all of them when every key is equal)
        uint32_t pmask = top_bit < 0 ? 0xffffffffu : (top_bit >= 31 ? 0u : ~((2u << top_bit) - 1u));
        uint32_t prefix = kmax & pmask, need = (uint32_t)kb;
#pragma unroll 1
        while (top_bit >= 0) {
            const int shift = max(0, top_bit - 10);
            const int nbins = 1 << (top_bit - shift + 1);
            top_bit = shift - 1;
            for (int i = tid; i < nbins; i += THREADS) hist[i] = 0u;
            __syncthreads();
            for (int t = tid; t < width; t += THREADS) {
                const uint32_t key = skey[t];
                if ((key & pmask) == prefix && srow[t] >= 0) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
            }
            __syncthreads();
            // the bins from the top, ceil(nbins / THREADS) a thread: the one holding the need-th key
            const int per = ceil_div(nbins, THREADS);
            const int top = nbins - 1 - tid * per;
            uint32_t mine = 0;
            for (int j = 0; j < per && top - j >= 0; ++j) mine += hist[top - j];
            uint32_t total;
            uint32_t run = mg_block_scan<W>(mine, s_ws, &total);
            for (int j = 0; j < per && top - j >= 0; ++j) {
                const uint32_t c = hist[top - j];
                if (run < need && run + c >= need) {
                    s_sel[0] = (uint32_t)(top - j);
                    s_sel[1] = run;
                }
                run += c;
            }
            __syncthreads();
            need -= s_sel[1];
            prefix |= s_sel[0] << shift;
            pmask |= (uint32_t)(nbins - 1) << shift;
            __syncthreads();  // s_sel and hist are free for the next pass
        }
        T = prefix;
        krem = need;  // >= 1: the keys equal to T to take, the first ones in row order
    }
    // chosen: every entry when kb == n, none when kb == 0, else key > T or one
    // of the first krem keys == T
    const bool all = kb == n, none = kb == 0;
    uint32_t eq = 0;
    if (!all && !none)
        for (int t = lo; t < hi; ++t) eq += srow[t] >= 0 && skey[t] == T;
    uint32_t eq_total;
    const uint32_t eq_ex = mg_block_scan<W>(eq, s_ws, &eq_total);
    auto chosen = [&](int t, uint32_t& e) -> bool {
        if (srow[t] < 0 || none) return false;
        if (all) return true;
        const uint32_t key = skey[t];
        const bool take = key > T || (key == T && e < krem);
        e += key == T;
        return take;
    };
    uint32_t sel = 0;
    {
        uint32_t e = eq_ex;
        for (int t = lo; t < hi; ++t) sel += chosen(t, e);
    }
    uint32_t sel_total;
    uint32_t pos = mg_block_scan<W>(sel, s_ws, &sel_total);
    {
        uint32_t e = eq_ex;
        for (int t = lo; t < hi; ++t)
            if (chosen(t, e)) {
                if (pos < (uint32_t)kb) out[pos] = srow[t];
                else atomicOr(flag, kFlagBounds);  // unreachable when the select is consistent
                ++pos;
            }
    }
    for (int p = kb + tid; p < k_max; p += THREADS) out[p] = -1;
}

__global__ void __launch_bounds__(kShThreads) merge_map_kernel(const int32_t* __restrict__ pos,
                                                              const int32_t* __restrict__ pk_rows, int width,
                                                              int k_max, int32_t* __restrict__ idx) {
    const int u = blockIdx.y, t = blockIdx.x * kShThreads + threadIdx.x;
    if (t >= k_max) return;
    const int p = pos[(size_t)u * k_max + t];
    idx[(size_t)u * k_max + t] = (p >= 0 && p < width) ? pk_rows[(size_t)u * width + p] : -1;
}

// the rows of the global list in [row0, row0 + rows_cap), as local rows at the
// front of the unit's list (they are one run of it: the list is ascending)
__global__ void __launch_bounds__(kShThreads) localize_kernel(const int32_t* __restrict__ idx, int k_max, int row0,
                                                             int rows_cap, int32_t* __restrict__ local) {
    __shared__ int s_red[33];
    const int u = blockIdx.y, tid = threadIdx.x;
    const int32_t* iu = idx + (size_t)u * k_max;
    int c = 0;
    for (int t = tid; t < k_max; t += kShThreads) c += iu[t] >= 0 && iu[t] < row0;
    const int lo = sh_block_sum(c, s_red);  // entries below this shard's rows
    const int t = blockIdx.x * kShThreads + tid;
    if (t >= k_max) return;
    const int src = lo + t;
    const int g = src < k_max ? iu[src] : -1;
    local[(size_t)u * k_max + t] = (g >= row0 && g - row0 < rows_cap) ? g - row0 : -1;
}

// one warp per (b, query head): lane l owns dims 4l..4l+3
__global__ void __launch_bounds__(32) shard_combine_kernel(const float* __restrict__ O_parts,
                                                          const float* __restrict__ lse_parts, int R, int heads,
                                                          float* __restrict__ O) {
    const int bh = blockIdx.x, lane = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, lse_parts[(size_t)r * heads + bh]);
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (M != -INFINITY) {
        for (int r = 0; r < R; ++r) {
            const float l = lse_parts[(size_t)r * heads + bh];
            if (l == -INFINITY) continue;
            const float w = exp2f(l - M);
            const float4 o = *reinterpret_cast<const float4*>(O_parts + ((size_t)r * heads + bh) * kD + 4 * lane);
            den += w;
            num.x += w * o.x;
            num.y += w * o.y;
            num.z += w * o.z;
            num.w += w * o.w;
        }
    }
    float4 out = make_float4(0.f, 0.f, 0.f, 0.f);
    if (den > 0.f) out = make_float4(num.x / den, num.y / den, num.z / den, num.w / den);
    *reinterpret_cast<float4*>(O + (size_t)bh * kD + 4 * lane) = out;
}

}  // namespace

cudaError_t launch_shard_pack(const float* scores, int rows_cap, int units, int k_max, int row0, int32_t* cand_rows,
                              float* cand_scores, unsigned* flag, cudaStream_t st) {
    if (units == 0 || k_max == 0) return cudaSuccess;
    shard_pack_kernel<<<dim3(ceil_div(k_max, kShThreads), units), kShThreads, 0, st>>>(scores, rows_cap, cand_rows,
                                                                                       cand_scores, k_max, row0, flag);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_merge_pack(const float* cand_scores, const int32_t* cand_rows, int R, int units, int Hkv,
                              int k_max, float* pk_scores, int32_t* pk_rows, int32_t* n_cand, uint32_t* hist,
                              unsigned* flag, cudaStream_t st) {
    if (units == 0) return cudaSuccess;
    if (k_max == 0) return cudaSuccess;
    merge_pack_kernel<<<dim3(ceil_div(R * k_max, kShThreads), units), kShThreads, 0, st>>>(
        cand_scores, cand_rows, R, units, Hkv, k_max, pk_scores, pk_rows, n_cand, hist, flag);
    note_launch();
    return cudaGetLastError();
}

bool merge_topk_fits(int R, int k_max) { return (long long)R * k_max <= kMergeCap; }

template <int THREADS>
static cudaError_t mg_launch(const float* cand_scores, const int32_t* cand_rows, int R, int units, int Hkv,
                             int k_max, const int32_t* kreq, int32_t* idx, unsigned* flag, cudaStream_t st) {
    static int configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(merge_topk_kernel<THREADS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMergeCap * 8);
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    merge_topk_kernel<THREADS><<<units, THREADS, (size_t)R * k_max * 8, st>>>(cand_scores, cand_rows, R, units, Hkv,
                                                                              k_max, kreq, idx, flag);
    return cudaGetLastError();
}

cudaError_t launch_merge_topk(const float* cand_scores, const int32_t* cand_rows, int R, int units, int Hkv,
                              int k_max, const int32_t* kreq, int32_t* idx, unsigned* flag, cudaStream_t st) {
    if (units == 0 || k_max == 0) return cudaSuccess;
    if (!merge_topk_fits(R, k_max)) return cudaErrorInvalidValue;
    // a few thousand candidates a unit: 1024 threads; short lists (many units):
    // 256, so that every unit's CTA is resident at once
    const cudaError_t e = R * k_max > 2048
        ? mg_launch<1024>(cand_scores, cand_rows, R, units, Hkv, k_max, kreq, idx, flag, st)
        : mg_launch<256>(cand_scores, cand_rows, R, units, Hkv, k_max, kreq, idx, flag, st);
    note_launch();
    return e;
}

cudaError_t launch_merge_map(const int32_t* pos, const int32_t* pk_rows, int units, int width, int k_max,
                             int32_t* idx, cudaStream_t st) {
    if (units == 0 || k_max == 0) return cudaSuccess;
    merge_map_kernel<<<dim3(ceil_div(k_max, kShThreads), units), kShThreads, 0, st>>>(pos, pk_rows, width, k_max,
                                                                                      idx);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_localize(const int32_t* idx, int units, int k_max, int row0, int rows_cap, int32_t* local,
                            cudaStream_t st) {
    if (units == 0 || k_max == 0) return cudaSuccess;
    localize_kernel<<<dim3(ceil_div(k_max, kShThreads), units), kShThreads, 0, st>>>(idx, k_max, row0, rows_cap,
                                                                                     local);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_shard_combine(const float* O_parts, const float* lse_parts, int R, int heads, float* O,
                                 cudaStream_t st) {
    if (heads == 0) return cudaSuccess;
    shard_combine_kernel<<<heads, 32, 0, st>>>(O_parts, lse_parts, R, heads, O);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tsa
