// overlap.cu -- exact overlap of the top-k index sets of several layers.
//
// HyLRA ("HyLRA: Hybrid Layer Reuse Attention", sec. 2.2) decides offline which
// layers may reuse an earlier layer's top-k from a lower-triangular matrix M of
// index-set overlap ratios between a source layer i and a target layer j >= i.
// This kernel counts |I_i(u) ∩ I_j(u)| for every pair of layers and every unit u
// from the index lists the decode steps wrote (ascending, then -1), and reduces
// the ratios |I_i ∩ I_j| / |I_j| over the units into M.
//
// One CTA per pair (i <= j).  Long lists (k_max > 256): the CTA walks the units
// in order, finding both lists' lengths (the first -1), checking their form,
// staging the source list in shared memory when it fits and looking every
// target entry up by binary search.  Short lists: each warp takes a unit at a
// time, both lists in its registers (lengths by ballots, look-ups by binary
// search over the source list in L1), and the CTA's barriers come once per 64
// units instead of four times a unit.  The counts are integers (exact); M sums
// the per-unit ratios in fp64 in unit order either way, so it is the same on
// every run.  Not a hot path: this is a profiling pass, run once per
// calibration batch.
#include "common.cuh"

namespace tsa {

namespace {

constexpr int kOvThreads = 256;
constexpr int kOvWarpK = 256;     // lists up to this long: a warp a unit
constexpr int kOvRound = 64;      // units a CTA holds ratios for between barriers (warp mode)
constexpr int kOvStage = 11776;  // source lists up to this length are staged (46 KB, under the 48 KB static limit)

// first position in [0, n) whose value is >= x (v ascending)
__device__ __forceinline__ int lower_bound(const int32_t* v, int n, int32_t x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (v[mid] < x)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

// warp mode: one warp's unit (lists a, b of k_max <= 256 entries): the target
// list's length, the overlap count and whether either list is malformed
__device__ __forceinline__ void warp_overlap(const int32_t* __restrict__ a, const int32_t* __restrict__ b, int k_max,
                                             int lane, int* na_out, int* nb_out, int* cnt_out, bool* bad_out) {
    constexpr int kM = kOvWarpK / 32;
    int32_t av[kM], bv[kM];
#pragma unroll
    for (int m = 0; m < kM; ++m) {
        const int t = 32 * m + lane;
        av[m] = t < k_max ? a[t] : -1;
        bv[m] = t < k_max ? b[t] : -1;
    }
    // lengths: the first negative entry (k_max when none)
    int na = k_max, nb = k_max;
#pragma unroll
    for (int m = kM - 1; m >= 0; --m) {
        const uint32_t ba = __ballot_sync(0xffffffffu, 32 * m + lane < k_max && av[m] < 0);
        const uint32_t bb = __ballot_sync(0xffffffffu, 32 * m + lane < k_max && bv[m] < 0);
        if (ba) na = 32 * m + __ffs(ba) - 1;
        if (bb) nb = 32 * m + __ffs(bb) - 1;
    }
    // the form: strictly ascending non-negative entries, then only -1
    bool bad = false;
#pragma unroll
    for (int m = 0; m < kM; ++m) {
        const int t = 32 * m + lane;
        int32_t an = __shfl_down_sync(0xffffffffu, av[m], 1), bn = __shfl_down_sync(0xffffffffu, bv[m], 1);
        if (m + 1 < kM) {
            const int32_t a0 = __shfl_sync(0xffffffffu, av[m + 1 < kM ? m + 1 : m], 0);
            const int32_t b0 = __shfl_sync(0xffffffffu, bv[m + 1 < kM ? m + 1 : m], 0);
            if (lane == 31) {
                an = a0;
                bn = b0;
            }
        }
        if (t < k_max) {
            bad |= t < na ? (t + 1 < na && av[m] >= an) : av[m] != -1;
            bad |= t < nb ? (t + 1 < nb && bv[m] >= bn) : bv[m] != -1;
        }
    }
    // each target entry looked up in the source list
    int c = 0;
#pragma unroll
    for (int m = 0; m < kM; ++m) {
        const int t = 32 * m + lane;
        if (t < nb) {
            const int pos = lower_bound(a, na, bv[m]);
            c += pos < na && a[pos] == bv[m];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    *na_out = na;
    *nb_out = nb;
    *cnt_out = c;
    *bad_out = __any_sync(0xffffffffu, bad);
}

__global__ void __launch_bounds__(kOvThreads) index_overlap_warp_kernel(const int32_t* __restrict__ idx, int L,
                                                                       int units, int k_max,
                                                                       int32_t* __restrict__ counts,
                                                                       double* __restrict__ M, unsigned* flag) {
    __shared__ double s_ratio[kOvRound];  // a unit's ratio, or -1 when its target list is empty
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p = blockIdx.x;
    int j = (int)((sqrt(8.0 * p + 1.0) - 1.0) * 0.5);
    while ((j + 1) * (j + 2) / 2 <= p) ++j;
    while (j * (j + 1) / 2 > p) --j;
    const int i = p - j * (j + 1) / 2;
    double sum = 0.0;  // thread 0
    int nonempty = 0;
    for (int u0 = 0; u0 < units; u0 += kOvRound) {
        for (int q = warp; q < kOvRound && u0 + q < units; q += kOvThreads / 32) {
            const int u = u0 + q;
            int na, nb, cnt;
            bool bad;
            warp_overlap(idx + ((size_t)i * units + u) * k_max, idx + ((size_t)j * units + u) * k_max, k_max, lane,
                         &na, &nb, &cnt, &bad);
            if (lane == 0) {
                if (counts) {
                    counts[((size_t)i * L + j) * units + u] = cnt;
                    counts[((size_t)j * L + i) * units + u] = cnt;
                }
                s_ratio[q] = nb > 0 ? (double)cnt / (double)nb : -1.0;
                if (bad) atomicOr(flag, kFlagBounds);
            }
        }
        __syncthreads();
        if (tid == 0)  // in unit order, as the walk of long lists sums them
            for (int q = 0; q < kOvRound && u0 + q < units; ++q)
                if (s_ratio[q] >= 0.0) {
                    sum += s_ratio[q];
                    ++nonempty;
                }
        __syncthreads();
    }
    if (tid == 0 && M) {
        M[(size_t)j * L + i] = nonempty > 0 ? sum / (double)nonempty : 1.0;
        if (i != j) M[(size_t)i * L + j] = 0.0;
    }
}

__global__ void __launch_bounds__(kOvThreads) index_overlap_kernel(const int32_t* __restrict__ idx, int L,
                                                                  int units, int k_max,
                                                                  int32_t* __restrict__ counts,
                                                                  double* __restrict__ M, unsigned* flag) {
    __shared__ int32_t s_src[kOvStage];
    __shared__ int s_na, s_nb, s_bad;
    __shared__ int s_red[kOvThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // pair p = j (j + 1) / 2 + i, i <= j
    const int p = blockIdx.x;
    int j = (int)((sqrt(8.0 * p + 1.0) - 1.0) * 0.5);
    while ((j + 1) * (j + 2) / 2 <= p) ++j;
    while (j * (j + 1) / 2 > p) --j;
    const int i = p - j * (j + 1) / 2;

    double sum = 0.0;  // thread 0: ratios of the units with a non-empty target list
    int nonempty = 0;
    for (int u = 0; u < units; ++u) {
        const int32_t* a = idx + ((size_t)i * units + u) * k_max;  // source
        const int32_t* b = idx + ((size_t)j * units + u) * k_max;  // target
        if (tid == 0) {
            s_na = k_max;
            s_nb = k_max;
            s_bad = 0;
        }
        __syncthreads();
        for (int t = tid; t < k_max; t += kOvThreads) {
            if (a[t] < 0) atomicMin(&s_na, t);
            if (b[t] < 0) atomicMin(&s_nb, t);
        }
        __syncthreads();
        const int na = s_na, nb = s_nb;
        // the form: strictly ascending non-negative entries, then only -1
        bool bad = false;
        for (int t = tid; t < k_max; t += kOvThreads) {
            const int32_t x = a[t], y = b[t];
            bad |= t < na ? (t + 1 < na && x >= a[t + 1]) : x != -1;
            bad |= t < nb ? (t + 1 < nb && y >= b[t + 1]) : y != -1;
            if (t < na && na <= kOvStage) s_src[t] = x;
        }
        if (bad) s_bad = 1;
        __syncthreads();
        const int32_t* src = na <= kOvStage ? s_src : a;
        int c = 0;
        for (int t = tid; t < nb; t += kOvThreads) {
            const int32_t y = b[t];
            const int pos = lower_bound(src, na, y);
            c += pos < na && src[pos] == y;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) s_red[warp] = c;
        __syncthreads();
        if (tid == 0) {
            int cnt = 0;
            for (int w = 0; w < kOvThreads / 32; ++w) cnt += s_red[w];
            if (counts) {
                counts[((size_t)i * L + j) * units + u] = cnt;
                counts[((size_t)j * L + i) * units + u] = cnt;
            }
            if (nb > 0) {
                sum += (double)cnt / (double)nb;
                ++nonempty;
            }
            if (s_bad) atomicOr(flag, kFlagBounds);
        }
        __syncthreads();  // shared state is reset for the next unit
    }
    if (tid == 0 && M) {
        M[(size_t)j * L + i] = nonempty > 0 ? sum / (double)nonempty : 1.0;
        if (i != j) M[(size_t)i * L + j] = 0.0;
    }
}

}  // namespace

cudaError_t launch_index_overlap(const int32_t* idx, int L, int units, int k_max, int32_t* counts, double* M,
                                 unsigned* flag, cudaStream_t st) {
    if (L == 0) return cudaSuccess;
    const int pairs = L * (L + 1) / 2;
    if (k_max <= kOvWarpK)
        index_overlap_warp_kernel<<<pairs, kOvThreads, 0, st>>>(idx, L, units, k_max, counts, M, flag);
    else
        index_overlap_kernel<<<pairs, kOvThreads, 0, st>>>(idx, L, units, k_max, counts, M, flag);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tsa
