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
