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
// Design: grid = (split, unit).  A CTA owns a contiguous range of the unit's
// index list.  Each half-warp gathers one 256-byte K row and one V row per step
// with 16-byte loads (8 dims per lane), so the 16 lanes of a half read a whole
// row; the g query heads of the kv-head stay in registers.  Logits go through a
// half-warp reduce-scatter and come back with a gather, then each lane updates
// the running (m, l, acc[8 dims]) of every head in the log2 domain.  The halves
// and warps are merged in shared memory, the CTA writes its partial
// (m, l, acc[128]) per head, and the last CTA of the unit to arrive (an atomic
// counter in the workspace, reset by that CTA) combines the partials into O.
#include "common.cuh"
#include "launch.h"

namespace tsa {

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kAttnTargetCtas = 4 * 148;  // split count aims at ~4 CTAs per SM
constexpr int kAttnMinRows = 32;           // at least this many positions per split
constexpr int kPartStride = kD + 2;        // m, l, acc[128]

template <int G>
__global__ void __launch_bounds__(kAttnThreads)
attn_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
            const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ lens,
            const int32_t* __restrict__ idx, const int32_t* __restrict__ kreq, int k_max,
            int block, int Hkv, int Ncap, float scale_log2, int S, float* __restrict__ part,
            unsigned* __restrict__ counters, float* __restrict__ O, unsigned* __restrict__ flag) {
    constexpr int R = 16 / G;
    constexpr int kRowsStep = 2 * R;
    const int s = blockIdx.x, unit = blockIdx.y;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = lane >> 4, c = lane & 15;

    int len = lens[b];
    if (len < 0 || len > Ncap) {
        if (tid == 0 && s == 0) atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    int npos, nb = 0;
    if (idx == nullptr) {
        npos = len;
    } else {
        nb = block == 1 ? len : ceil_div(len, block);
        int kb = kreq ? kreq[b] : k_max;
        kb = max(0, min(kb, nb));
        if (kb > k_max) {
            if (tid == 0 && s == 0) atomicOr(flag, kFlagBounds);
            kb = k_max;
        }
        npos = kb * block;
    }
    const int chunk = ceil_div(npos, S);
    const int p0 = min(s * chunk, npos), p1 = min(p0 + chunk, npos);

    float q[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        unpack8(*reinterpret_cast<const uint4*>(Q + ((size_t)unit * G + h) * kD + 8 * c), q[h]);
#pragma unroll
        for (int e = 0; e < 8; ++e) q[h][e] *= scale_log2;
    }
    float m[G], l[G], acc[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
    }
    const int32_t* iu = idx ? idx + (size_t)unit * k_max : nullptr;
    const __nv_bfloat16* kbase = K + (size_t)unit * Ncap * kD + 8 * c;
    const __nv_bfloat16* vbase = V + (size_t)unit * Ncap * kD + 8 * c;

    for (int base = p0 + warp * kRowsStep; base < p1; base += kAttnWarps * kRowsStep) {
        int rows[R];
        uint4 kr[R], vr[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int pos = base + 2 * r + half;
            int row = -1;
            if (pos < p1) {
                if (iu == nullptr) {
                    row = pos;
                } else if (block == 1) {
                    row = iu[pos];
                    if (row >= len) {
                        atomicOr(flag, kFlagBounds);
                        row = -1;
                    }
                } else {
                    const int slot = pos / block;
                    const int e = iu[slot];
                    if (e >= nb) {
                        atomicOr(flag, kFlagBounds);
                    } else if (e >= 0) {
                        row = e * block + (pos - slot * block);
                        if (row >= len) row = -1;  // tail of a partial last block
                    }
                }
            }
            rows[r] = row < 0 ? -1 : row;
            kr[r] = row >= 0 ? ld_stream(kbase + (size_t)row * kD) : make_uint4(0, 0, 0, 0);
            vr[r] = row >= 0 ? ld_stream(vbase + (size_t)row * kD) : make_uint4(0, 0, 0, 0);
        }
        float v[16];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float kf[8];
            unpack8(kr[r], kf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float d = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) d = fmaf(kf[e], q[h][e], d);
                v[r * G + h] = d;
            }
        }
        halfwarp_reduce_scatter16(v, c);
        float z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = __shfl_sync(0xffffffffu, v[0], (lane & 16) | i);
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (rows[r] < 0)
#pragma unroll
                for (int h = 0; h < G; ++h) z[r * G + h] = -INFINITY;
        float vf[R][8];
#pragma unroll
        for (int r = 0; r < R; ++r) unpack8(vr[r], vf[r]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float mt = m[h];
#pragma unroll
            for (int r = 0; r < R; ++r) mt = fmaxf(mt, z[r * G + h]);
            if (mt == -INFINITY) continue;  // no valid row for this head yet
            const float alpha = exp2f(m[h] - mt);  // 0 when m[h] = -inf
            l[h] *= alpha;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h][e] *= alpha;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float p = exp2f(z[r * G + h] - mt);  // 0 for skipped rows
                l[h] += p;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[h][e] = fmaf(p, vf[r][e], acc[h][e]);
            }
            m[h] = mt;
        }
    }

    // merge the two halves of the warp (lane c and lane c+16 hold the same dims)
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[h], 16);
        const float lo = __shfl_xor_sync(0xffffffffu, l[h], 16);
        float ao[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ao[e] = __shfl_xor_sync(0xffffffffu, acc[h][e], 16);
        const float mn = fmaxf(m[h], mo);
        if (mn != -INFINITY) {
            const float a = exp2f(m[h] - mn), ab = exp2f(mo - mn);
            l[h] = l[h] * a + lo * ab;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h][e] = acc[h][e] * a + ao[e] * ab;
            m[h] = mn;
        }
    }
    __shared__ float s_m[kAttnWarps][G], s_l[kAttnWarps][G];
    __shared__ float s_acc[kAttnWarps][G][kD];
    if (half == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int e = 0; e < 8; ++e) s_acc[warp][h][8 * c + e] = acc[h][e];
            if (c == 0) {
                s_m[warp][h] = m[h];
                s_l[warp][h] = l[h];
            }
        }
    }
    __syncthreads();
    // thread t = dimension t: merge the warps and write this split's partial
    float* pu = part + ((size_t)unit * S + s) * G * kPartStride;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w][h]);
        float A = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kAttnWarps; ++w) {
                if (s_m[w][h] == -INFINITY) continue;
                const float sc = exp2f(s_m[w][h] - M);
                A += s_acc[w][h][tid] * sc;
                L += s_l[w][h] * sc;
            }
        }
        pu[h * kPartStride + 2 + tid] = A;
        if (tid == 0) {
            pu[h * kPartStride] = M;
            pu[h * kPartStride + 1] = L;
        }
    }

    // the last CTA of this unit to arrive combines all splits
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&counters[unit], 1u) == (unsigned)(S - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float* pall = part + (size_t)unit * S * G * kPartStride;
#pragma unroll 1
    for (int h = 0; h < G; ++h) {
        float M = -INFINITY;
        for (int j = 0; j < S; ++j) M = fmaxf(M, __ldcg(pall + ((size_t)j * G + h) * kPartStride));
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
            for (int j = 0; j < S; ++j) {
                const float* pj = pall + ((size_t)j * G + h) * kPartStride;
                const float mj = __ldcg(pj);
                if (mj == -INFINITY) continue;
                const float w = exp2f(mj - M);
                den += w * __ldcg(pj + 1);
                num += w * __ldcg(pj + 2 + tid);
            }
        }
        O[((size_t)unit * G + h) * kD + tid] = den > 0.f ? num / den : 0.f;
    }
    if (tid == 0) counters[unit] = 0u;  // ready for the next launch on this workspace
}

int attn_splits(const Dims& d, int k_max, int block, bool dense) {
    long long rows;
    if (dense) {
        rows = d.Ncap;
    } else {
        const long long nbmax = block == 1 ? d.Ncap : ceil_div(d.Ncap, block);
        rows = (long long)(k_max < nbmax ? k_max : nbmax) * block;
    }
    const int units = d.units() > 0 ? d.units() : 1;
    int s = ceil_div(kAttnTargetCtas, units);
    const long long smax = (rows + kAttnMinRows - 1) / kAttnMinRows;
    if (s > smax) s = (int)smax;
    if (s > 1024) s = 1024;
    if (s < 1) s = 1;
    return s;
}

size_t attn_partials_floats(const Dims& d, int splits) {
    return (size_t)d.units() * splits * d.G * kPartStride;
}

cudaError_t launch_attn(const void* Q, const void* K, const void* V, const int32_t* lens,
                        const int32_t* idx, const int32_t* kreq, int k_max, int block,
                        const Dims& d, float scale, int splits, float* partials,
                        unsigned* counters, float* O, unsigned* flag, cudaStream_t st) {
    if (d.units() == 0) return cudaSuccess;
    dim3 grid(splits, d.units());
    const float sl2 = scale * kLog2e;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
    const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(K);
    const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(V);
#define TSA_ATTN_CASE(g)                                                                        \
    case g:                                                                                     \
        attn_kernel<g><<<grid, kAttnThreads, 0, st>>>(q, k, v, lens, idx, kreq, k_max, block,    \
                                                      d.Hkv, d.Ncap, sl2, splits, partials,     \
                                                      counters, O, flag);                       \
        break;
    switch (d.G) {
        TSA_ATTN_CASE(1)
        TSA_ATTN_CASE(2)
        TSA_ATTN_CASE(4)
        TSA_ATTN_CASE(8)
        default:
            return cudaErrorInvalidValue;
    }
#undef TSA_ATTN_CASE
    note_launch();
    return cudaGetLastError();
}

}  // namespace tsa
