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

__global__ void __launch_bounds__(kShThreads) shard_pack_kernel(const float* __restrict__ scores, int rows_cap,
                                                               int32_t* __restrict__ cand_rows,
                                                               float* __restrict__ cand_scores, int k_max,
                                                               int row0, unsigned* flag) {
    const int u = blockIdx.x;
    for (int t = threadIdx.x; t < k_max; t += kShThreads) {
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
}

// one CTA per unit: the candidates of shards 0..R-1 (each a list of valid rows,
// then -1) packed one after another, then padded with (-inf, -1)
__global__ void __launch_bounds__(kShThreads) merge_pack_kernel(const float* __restrict__ cand_scores,
                                                               const int32_t* __restrict__ cand_rows, int R,
                                                               int units, int Hkv, int k_max,
                                                               float* __restrict__ pk_scores,
                                                               int32_t* __restrict__ pk_rows,
                                                               int32_t* __restrict__ n_cand, unsigned* flag) {
    __shared__ int s_cnt[kMaxShards + 1];
    const int u = blockIdx.x, tid = threadIdx.x;
    const int width = R * k_max;
    for (int r = tid; r <= R; r += kShThreads) s_cnt[r] = k_max;
    __syncthreads();
    for (int r = 0; r < R; ++r) {
        const int32_t* cr = cand_rows + ((size_t)r * units + u) * k_max;
        for (int t = tid; t < k_max; t += kShThreads)
            if (cr[t] < 0) atomicMin(&s_cnt[r], t);
    }
    __syncthreads();
    if (tid == 0) {  // counts -> offsets; the shards must come in row order
        int off = 0, last = -1;
        for (int r = 0; r < R; ++r) {
            const int c = s_cnt[r];
            const int32_t* cr = cand_rows + ((size_t)r * units + u) * k_max;
            if (c > 0) {
                if (cr[0] <= last) atomicOr(flag, kFlagBounds);
                last = cr[c - 1];
            }
            s_cnt[r] = off;
            off += c;
        }
        s_cnt[R] = off;
        if (u % Hkv == 0) n_cand[u / Hkv] = off;  // the same for every kv-head of a sequence
    }
    __syncthreads();
    float* ps = pk_scores + (size_t)u * width;
    int32_t* pr = pk_rows + (size_t)u * width;
    for (int r = 0; r < R; ++r) {
        const int off = s_cnt[r], c = s_cnt[r + 1] - off;
        const float* cs = cand_scores + ((size_t)r * units + u) * k_max;
        const int32_t* cr = cand_rows + ((size_t)r * units + u) * k_max;
        for (int t = tid; t < c; t += kShThreads) {
            ps[off + t] = cs[t];
            pr[off + t] = cr[t];
        }
    }
    for (int t = s_cnt[R] + tid; t < width; t += kShThreads) {
        ps[t] = -INFINITY;
        pr[t] = -1;
    }
}

__global__ void __launch_bounds__(kShThreads) merge_map_kernel(const int32_t* __restrict__ pos,
                                                              const int32_t* __restrict__ pk_rows, int width,
                                                              int k_max, int32_t* __restrict__ idx) {
    const int u = blockIdx.x;
    for (int t = threadIdx.x; t < k_max; t += kShThreads) {
        const int p = pos[(size_t)u * k_max + t];
        idx[(size_t)u * k_max + t] = (p >= 0 && p < width) ? pk_rows[(size_t)u * width + p] : -1;
    }
}

// the rows of the global list in [row0, row0 + rows_cap), as local rows at the
// front of the unit's list (they are one run of it: the list is ascending)
__global__ void __launch_bounds__(kShThreads) localize_kernel(const int32_t* __restrict__ idx, int k_max, int row0,
                                                             int rows_cap, int32_t* __restrict__ local) {
    __shared__ int s_lo;
    const int u = blockIdx.x, tid = threadIdx.x;
    const int32_t* iu = idx + (size_t)u * k_max;
    if (tid == 0) s_lo = 0;
    __syncthreads();
    int c = 0;
    for (int t = tid; t < k_max; t += kShThreads) c += iu[t] >= 0 && iu[t] < row0;
    if (c) atomicAdd(&s_lo, c);
    __syncthreads();
    const int lo = s_lo;
    for (int t = tid; t < k_max; t += kShThreads) {
        const int src = lo + t;
        const int g = src < k_max ? iu[src] : -1;
        local[(size_t)u * k_max + t] = (g >= row0 && g - row0 < rows_cap) ? g - row0 : -1;
    }
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
    shard_pack_kernel<<<units, kShThreads, 0, st>>>(scores, rows_cap, cand_rows, cand_scores, k_max, row0, flag);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_merge_pack(const float* cand_scores, const int32_t* cand_rows, int R, int units, int Hkv,
                              int k_max, float* pk_scores, int32_t* pk_rows, int32_t* n_cand, unsigned* flag,
                              cudaStream_t st) {
    if (units == 0) return cudaSuccess;
    merge_pack_kernel<<<units, kShThreads, 0, st>>>(cand_scores, cand_rows, R, units, Hkv, k_max, pk_scores, pk_rows,
                                                    n_cand, flag);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_merge_map(const int32_t* pos, const int32_t* pk_rows, int units, int width, int k_max,
                             int32_t* idx, cudaStream_t st) {
    if (units == 0 || k_max == 0) return cudaSuccess;
    merge_map_kernel<<<units, kShThreads, 0, st>>>(pos, pk_rows, width, k_max, idx);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_localize(const int32_t* idx, int units, int k_max, int row0, int rows_cap, int32_t* local,
                            cudaStream_t st) {
    if (units == 0 || k_max == 0) return cudaSuccess;
    localize_kernel<<<units, kShThreads, 0, st>>>(idx, k_max, row0, rows_cap, local);
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
