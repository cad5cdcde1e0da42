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
// index list and walks it in tiles of 64 rows.  The rows' K and V (256 B each)
// are gathered into shared memory with 16-byte cp.async copies (a 3-stage ring
// when the range spans several tiles, one stage when it fits in one tile, so
// that short sparse ranges leave room for more CTAs per SM).  Per tile, with
// tile-level online softmax:
//   A. logits: each half-warp owns 4 rows of the tile, each lane 8 dims; the g
//      query heads stay in registers; partial dots are reduce-scattered across
//      the half-warp and written to shared memory as z[row][head] (log2 units);
//   B. one warp per head takes the tile max, the running max M, the rescale
//      factor of the accumulators and p = 2^(z - M), and updates the running
//      sum L;
//   C. each lane accumulates p * V for its 8 dims and every head (no per-row
//      rescaling, no cross-lane traffic).
// Halves and warps are merged at the end into the CTA's partial (M, L,
// acc[128]) per head.  With at most 16 splits per unit the splits of a unit
// form one thread-block cluster and combine through distributed shared memory
// (no scratch).  With more (few units, long ranges) each CTA writes its partial
// to the workspace and the last CTA of the unit to arrive (an atomic counter in
// the workspace, reset by that CTA) combines the partials into O.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace tsa {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kTileRows = 64;                         // rows per staged tile
constexpr int kRowGroups = kAttnThreads / 16;         // half-warps: 16
constexpr int kRowsPerGroup = kTileRows / kRowGroups; // 4 rows of a tile per half-warp
constexpr int kStageBytes = kTileRows * kD * 2 * 2;   // K and V of one tile (32 KB)
constexpr int kMaxSplits = 256;
constexpr int kClusterMax = 16;  // splits per unit that combine inside one cluster
constexpr int kSms = 148;
constexpr int kPartStride = kD + 4;  // M, L, 2 pad, acc[128]: 528 B, 16-byte aligned

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__host__ __device__ constexpr int attn_smem_bytes(int G, int stages) {
    return stages * kStageBytes > kAttnWarps * G * kD * 4 ? stages * kStageBytes : kAttnWarps * G * kD * 4;
}

template <int G, int STAGES, bool CLUSTER>
__global__ void __launch_bounds__(kAttnThreads, G >= 8 ? 1 : 2)
attn_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
            const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ lens,
            const int32_t* __restrict__ idx, const int32_t* __restrict__ kreq, int k_max,
            int block, int Hkv, int Ncap, float scale_log2, int S, float* __restrict__ part,
            unsigned* __restrict__ counters, float* __restrict__ O, unsigned* __restrict__ flag) {
    constexpr int R = 16 / G;  // rows per half-warp per logit pass (R*G = 16 partial dots)
    constexpr int kPassesA = (kRowsPerGroup + R - 1) / R;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_row[STAGES][kTileRows];
    __shared__ __align__(16) float s_z[kTileRows][G];  // logits, then weights p
    __shared__ float s_M[G], s_L[G], s_alpha[G];
    __shared__ float s_m[kAttnWarps][G], s_l[kAttnWarps][G];
    __shared__ float s_cm[kMaxSplits * G], s_cl[kMaxSplits * G];
    __shared__ __align__(16) float s_part[G][kD];  // the cluster path's partial
    __shared__ int s_last;

    const int s = blockIdx.x, unit = blockIdx.y;
    const int b = unit / Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = lane >> 4, c = lane & 15;
    const int rg = tid >> 4;  // this half-warp's row group

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
    const int ntiles = ceil_div(p1 - p0, kTileRows);
    const int32_t* iu = idx ? idx + (size_t)unit * k_max : nullptr;
    const __nv_bfloat16* Ku = K + (size_t)unit * Ncap * kD;
    const __nv_bfloat16* Vu = V + (size_t)unit * Ncap * kD;

    // cache row of position pos, or -1 (skipped entry, tail of a partial block)
    auto row_of = [&](int pos) -> int {
        if (iu == nullptr) return pos;
        if (block == 1) {
            const int r = iu[pos];
            if (r >= len) {
                atomicOr(flag, kFlagBounds);
                return -1;
            }
            return r < 0 ? -1 : r;
        }
        const int slot = pos / block;
        const int e = iu[slot];
        if (e >= nb) {
            atomicOr(flag, kFlagBounds);
            return -1;
        }
        if (e < 0) return -1;
        const int r = e * block + (pos - slot * block);
        return r < len ? r : -1;
    };
    // stage tile t: thread (slot = tid/4, quarter = tid%4) copies 64 B of K and 64 B of V
    auto issue = [&](int t) {
        if (t < ntiles) {
            const int st = t % STAGES;
            const int slot = tid >> 2, q4 = tid & 3;
            const int pos = p0 + t * kTileRows + slot;
            const int row = pos < p1 ? row_of(pos) : -1;
            if (q4 == 0) s_row[st][slot] = row;
            if (row >= 0) {
                unsigned char* kd = smem + st * kStageBytes + slot * (kD * 2) + q4 * 64;
                unsigned char* vd = kd + kTileRows * kD * 2;
                const unsigned char* ks = reinterpret_cast<const unsigned char*>(Ku + (size_t)row * kD) + q4 * 64;
                const unsigned char* vs = reinterpret_cast<const unsigned char*>(Vu + (size_t)row * kD) + q4 * 64;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    cp_async16(kd + 16 * j, ks + 16 * j);
                    cp_async16(vd + 16 * j, vs + 16 * j);
                }
            }
        }
        cp_async_commit();  // one group per tile slot, empty past the end: uniform accounting
    };

    float q[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        unpack8(*reinterpret_cast<const uint4*>(Q + ((size_t)unit * G + h) * kD + 8 * c), q[h]);
#pragma unroll
        for (int e = 0; e < 8; ++e) q[h][e] *= scale_log2;
    }
    float acc[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
    if (tid < G) {
        s_M[tid] = -INFINITY;
        s_L[tid] = 0.f;
    }

#pragma unroll
    for (int t = 0; t < STAGES - 1; ++t) issue(t);
    for (int t = 0; t < ntiles; ++t) {
        issue(t + STAGES - 1);
        cp_async_wait<STAGES - 1>();
        __syncthreads();
        const int st = t % STAGES;
        const int tile_rows = min(kTileRows, p1 - p0 - t * kTileRows);
        const unsigned char* ks = smem + st * kStageBytes;
        const unsigned char* vs = ks + kTileRows * kD * 2;

        // A. logits z[slot][h] for this half-warp's rows
#pragma unroll
        for (int pa = 0; pa < kPassesA; ++pa) {
            bool ok[R];
            uint4 kr[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int slot = rg + kRowGroups * (pa * R + r);
                ok[r] = slot < tile_rows && s_row[st][slot] >= 0;
                kr[r] = ok[r] ? *reinterpret_cast<const uint4*>(ks + slot * (kD * 2) + 16 * c) : make_uint4(0, 0, 0, 0);
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
            halfwarp_reduce_scatter16(v, c);  // lane c: row pa*R + c/G of the group, head c%G
            const int r = c / G, h = c - (c / G) * G;
            const int slot = rg + kRowGroups * (pa * R + r);
            if (slot < kTileRows) {
                const bool valid = slot < tile_rows && s_row[st][slot] >= 0;
                s_z[slot][h] = valid ? v[0] : -INFINITY;
            }
        }
        __syncthreads();
        // B. warp h: tile max, running max and sum, weights p = 2^(z - M)
        if (warp < G) {
            const int h = warp;
            const float z0 = s_z[lane][h], z1 = s_z[lane + 32][h];
            float mt = fmaxf(z0, z1);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
            const float Mold = s_M[h];
            const float Mnew = fmaxf(Mold, mt);
            const float alpha = Mold == -INFINITY ? 0.f : exp2f(Mold - Mnew);
            const float p0v = z0 == -INFINITY ? 0.f : exp2f(z0 - Mnew);
            const float p1v = z1 == -INFINITY ? 0.f : exp2f(z1 - Mnew);
            s_z[lane][h] = p0v;
            s_z[lane + 32][h] = p1v;
            float ps = p0v + p1v;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            if (lane == 0) {
                s_M[h] = Mnew;
                s_L[h] = s_L[h] * alpha + ps;
                s_alpha[h] = alpha;
            }
        }
        __syncthreads();
        // C. acc[h][8 dims] = alpha_h * acc + sum over this group's rows of p[row][h] * V[row]
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float a = s_alpha[h];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h][e] *= a;
        }
#pragma unroll
        for (int i = 0; i < kRowsPerGroup; ++i) {
            const int slot = rg + kRowGroups * i;
            if (slot >= tile_rows || s_row[st][slot] < 0) continue;
            float vf[8];
            unpack8(*reinterpret_cast<const uint4*>(vs + slot * (kD * 2) + 16 * c), vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float p = s_z[slot][h];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[h][e] = fmaf(p, vf[e], acc[h][e]);
            }
        }
        __syncthreads();  // this stage and s_z are refilled next iteration
    }
    cp_async_wait<0>();

    // merge the two halves of each warp, then the warps (all share the CTA's M)
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], 16);
    __syncthreads();
    float* s_acc = reinterpret_cast<float*>(smem);  // [kAttnWarps][G][128]
    if (half == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float* dst = s_acc + (warp * G + h) * kD + 8 * c;
            *reinterpret_cast<float4*>(dst) = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
            *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
        }
    }
    __syncthreads();
    if (tid < G * 32) {  // thread (h, quad): dims 4*quad..4*quad+3 of head h
        const int h = tid >> 5, qd = tid & 31;
        float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            const float4 a = *reinterpret_cast<const float4*>(s_acc + (w * G + h) * kD + 4 * qd);
            A.x += a.x;
            A.y += a.y;
            A.z += a.z;
            A.w += a.w;
        }
        if constexpr (CLUSTER) {
            *reinterpret_cast<float4*>(&s_part[h][4 * qd]) = A;
        } else {
            float* pu = part + (((size_t)unit * S + s) * G + h) * kPartStride;
            *reinterpret_cast<float4*>(pu + 4 + 4 * qd) = A;
            if (qd == 0) *reinterpret_cast<float2*>(pu) = make_float2(s_M[h], s_L[h]);
        }
    }

    if constexpr (CLUSTER) {
        // the S splits of this unit are the S CTAs of this cluster (rank = split)
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();  // every partial (s_M, s_L, s_part) is complete
        const int per = (G * 32 + S - 1) / S;  // float4 output slots per CTA
        if (tid < per) {
            const int slot = s * per + tid;
            if (slot < G * 32) {
                const int h = slot >> 5, qd = slot & 31;
                float mj[kClusterMax], lj[kClusterMax];
                float M = -INFINITY;
#pragma unroll
                for (int j = 0; j < kClusterMax; ++j) {
                    mj[j] = -INFINITY;
                    lj[j] = 0.f;
                    if (j < S) {
                        mj[j] = *cluster.map_shared_rank(&s_M[h], j);
                        lj[j] = *cluster.map_shared_rank(&s_L[h], j);
                    }
                    M = fmaxf(M, mj[j]);
                }
                float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
                float den = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int j = 0; j < kClusterMax; ++j) {
                        if (j >= S) break;
                        const float w = mj[j] == -INFINITY ? 0.f : exp2f(mj[j] - M);
                        const float4 o = *reinterpret_cast<const float4*>(cluster.map_shared_rank(&s_part[h][4 * qd], j));
                        den += w * lj[j];
                        num.x += w * o.x;
                        num.y += w * o.y;
                        num.z += w * o.z;
                        num.w += w * o.w;
                    }
                }
                float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
                if (den > 0.f) r = make_float4(num.x / den, num.y / den, num.z / den, num.w / den);
                *reinterpret_cast<float4*>(O + ((size_t)unit * G + h) * kD + 4 * qd) = r;
            }
        }
        cluster.sync();  // no CTA leaves while another may still read its shared memory
        return;
    }

    // the last CTA of this unit to arrive combines all splits
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&counters[unit], 1u) == (unsigned)(S - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float* pall = part + (size_t)unit * S * G * kPartStride;
    for (int i = tid; i < S * G; i += kAttnThreads) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(pall + (size_t)i * kPartStride));
        s_cm[i] = ml.x;
        s_cl[i] = ml.y;
    }
    __syncthreads();
    if (tid < G * 32) {
        const int h = tid >> 5, qd = tid & 31;
        float M = -INFINITY;
        for (int j = 0; j < S; ++j) M = fmaxf(M, s_cm[j * G + h]);
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
        float den = 0.f;
        if (M != -INFINITY) {
#pragma unroll 8
            for (int j = 0; j < S; ++j) {
                const float mj = s_cm[j * G + h];
                const float w = mj == -INFINITY ? 0.f : exp2f(mj - M);
                const float4 o = __ldcg(reinterpret_cast<const float4*>(pall + ((size_t)j * G + h) * kPartStride + 4 + 4 * qd));
                den += w * s_cl[j * G + h];
                num.x += w * o.x;
                num.y += w * o.y;
                num.z += w * o.z;
                num.w += w * o.w;
            }
        }
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
        if (den > 0.f) r = make_float4(num.x / den, num.y / den, num.z / den, num.w / den);
        *reinterpret_cast<float4*>(O + ((size_t)unit * G + h) * kD + 4 * qd) = r;
    }
    if (tid == 0) counters[unit] = 0u;  // ready for the next launch on this workspace
}

int attn_splits(const Dims& d, int k_max, int block, bool dense) {
    const int units = d.units() > 0 ? d.units() : 1;
    long long rows;
    int s;
    if (dense) {
        rows = d.Ncap;
        s = ceil_div(2 * kSms, units);  // one wave at two CTAs per SM
    } else {
        const long long nbmax = block == 1 ? d.Ncap : ceil_div(d.Ncap, block);
        rows = (long long)(k_max < nbmax ? k_max : nbmax) * block;
        s = (int)((rows + kTileRows - 1) / kTileRows);  // one tile per split where possible
    }
    // Up to 16 splits combine inside a cluster (no scratch round trip).  Past 16,
    // stay at 16 unless that leaves most of the GPU idle (fewer than 4 units).
    if (s > kClusterMax && units * kClusterMax >= 4 * kClusterMax) s = kClusterMax;
    const long long smax = (rows + 31) / 32;  // at least 32 positions per split
    if (s > smax) s = (int)smax;
    if (s > kMaxSplits) s = kMaxSplits;
    if (s < 1) s = 1;
    return s;
}

size_t attn_partials_floats(const Dims& d, int splits) {
    return (size_t)d.units() * splits * d.G * kPartStride;
}

static int g_attn_configured[64];

bool attn_uses_cluster(int splits) { return splits <= kClusterMax; }

template <int G, int STAGES, bool CLUSTER>
static cudaError_t attn_launch_g(dim3 grid, cudaStream_t st, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                 const __nv_bfloat16* v, const int32_t* lens, const int32_t* idx,
                                 const int32_t* kreq, int k_max, int block, const Dims& d, float sl2,
                                 int splits, float* partials, unsigned* counters, float* O, unsigned* flag) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = attn_smem_bytes(G, STAGES);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CLUSTER ? (unsigned)splits : 1u;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_kernel<G, STAGES, CLUSTER>, q, k, v, lens, idx, kreq, k_max, block,
                              d.Hkv, d.Ncap, sl2, splits, partials, counters, O, flag);
}

template <int G, int STAGES, bool CLUSTER>
static cudaError_t attn_configure_one() {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<G, STAGES, CLUSTER>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes(G, STAGES));
    if (e == cudaSuccess && CLUSTER)
        e = cudaFuncSetAttribute(attn_kernel<G, STAGES, CLUSTER>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

template <int G>
static cudaError_t attn_configure() {
    cudaError_t e = attn_configure_one<G, 1, true>();
    if (e == cudaSuccess) e = attn_configure_one<G, 3, true>();
    if (e == cudaSuccess) e = attn_configure_one<G, 1, false>();
    if (e == cudaSuccess) e = attn_configure_one<G, 3, false>();
    return e;
}

template <int G>
static cudaError_t attn_dispatch(bool one_tile, bool cluster, dim3 grid, cudaStream_t st, const __nv_bfloat16* q,
                                 const __nv_bfloat16* k, const __nv_bfloat16* v, const int32_t* lens,
                                 const int32_t* idx, const int32_t* kreq, int k_max, int block, const Dims& d,
                                 float sl2, int splits, float* partials, unsigned* counters, float* O,
                                 unsigned* flag) {
    if (cluster) {
        if (one_tile)
            return attn_launch_g<G, 1, true>(grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits,
                                             partials, counters, O, flag);
        return attn_launch_g<G, 3, true>(grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits,
                                         partials, counters, O, flag);
    }
    if (one_tile)
        return attn_launch_g<G, 1, false>(grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits,
                                          partials, counters, O, flag);
    return attn_launch_g<G, 3, false>(grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits, partials,
                                      counters, O, flag);
}

cudaError_t launch_attn(const void* Q, const void* K, const void* V, const int32_t* lens,
                        const int32_t* idx, const int32_t* kreq, int k_max, int block,
                        const Dims& d, float scale, int splits, float* partials,
                        unsigned* counters, float* O, unsigned* flag, cudaStream_t st) {
    if (d.units() == 0) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !g_attn_configured[dev]) {
        if ((e = attn_configure<1>()) != cudaSuccess) return e;
        if ((e = attn_configure<2>()) != cudaSuccess) return e;
        if ((e = attn_configure<4>()) != cudaSuccess) return e;
        if ((e = attn_configure<8>()) != cudaSuccess) return e;
        g_attn_configured[dev] = 1;
    }
    // positions per split (an upper bound): one tile -> single-stage kernel
    long long rows;
    if (idx == nullptr) {
        rows = d.Ncap;
    } else {
        const long long nbmax = block == 1 ? d.Ncap : ceil_div(d.Ncap, block);
        rows = (long long)(k_max < nbmax ? k_max : nbmax) * block;
    }
    const bool one_tile = (rows + splits - 1) / splits <= kTileRows;
    const bool cluster = attn_uses_cluster(splits);
    dim3 grid(splits, d.units());
    const float sl2 = scale * kLog2e;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q);
    const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(K);
    const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(V);
    switch (d.G) {
        case 1: e = attn_dispatch<1>(one_tile, cluster, grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits, partials, counters, O, flag); break;
        case 2: e = attn_dispatch<2>(one_tile, cluster, grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits, partials, counters, O, flag); break;
        case 4: e = attn_dispatch<4>(one_tile, cluster, grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits, partials, counters, O, flag); break;
        case 8: e = attn_dispatch<8>(one_tile, cluster, grid, st, q, k, v, lens, idx, kreq, k_max, block, d, sl2, splits, partials, counters, O, flag); break;
        default: return cudaErrorInvalidValue;
    }
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tsa
