// api.cu -- the C ABI of libtsa (declared in include/tsa.h): argument checks,
// workspace layout and stream-ordered launches.  No allocation, no
// synchronisation (except tsa_check_device_status), no exceptions.
#include <atomic>
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "launch.h"
#include "tsa.h"

namespace tsa {
static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace tsa

namespace {

thread_local char g_err[512] = "";

tsa_status fail(tsa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

}  // namespace

namespace tsa {
void set_error_message(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }
}  // namespace tsa

namespace {

tsa_status cuda_fail(cudaError_t e, const char* where) {
    return fail(TSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tsa_status check_shape(const tsa_shape& s, tsa::Dims* d) {
    if (s.B < 0 || s.Hq <= 0 || s.Hkv <= 0 || s.Ncap < 0)
        return fail(TSA_ERR_INVALID_ARG, "shape: need B >= 0, Hq > 0, Hkv > 0, Ncap >= 0 (got B=%d Hq=%d Hkv=%d Ncap=%d)",
                    s.B, s.Hq, s.Hkv, s.Ncap);
    if (s.d != tsa::kDHead) return fail(TSA_ERR_UNSUPPORTED, "shape: head dimension must be 128 (got %d)", s.d);
    if (s.Hq % s.Hkv != 0) return fail(TSA_ERR_INVALID_ARG, "shape: Hq=%d is not a multiple of Hkv=%d", s.Hq, s.Hkv);
    const int G = s.Hq / s.Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return fail(TSA_ERR_UNSUPPORTED, "shape: GQA group Hq/Hkv=%d not in {1,2,4,8}", G);
    if ((long long)s.B * s.Hkv > 65535)
        return fail(TSA_ERR_UNSUPPORTED, "shape: B*Hkv=%lld above 65535", (long long)s.B * s.Hkv);
    d->B = s.B;
    d->Hq = s.Hq;
    d->Hkv = s.Hkv;
    d->Ncap = s.Ncap;
    d->G = G;
    return TSA_OK;
}

tsa_status check_block(int block) {
    if (block < 1 || block > 4096) return fail(TSA_ERR_INVALID_ARG, "block must be in [1, 4096] (got %d)", block);
    return TSA_OK;
}

tsa_status check_scale(float scale) {
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(TSA_ERR_INVALID_ARG, "scale must be finite and > 0 (got %g)", (double)scale);
    return TSA_OK;
}

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

constexpr size_t kFlagBytes = 256;

// Workspace: [flag 256 B][top-digit histograms][split counters][split partials]
// [scores (SELECT, and FULL handing on its top-k)]
struct Layout {
    size_t counters = 0, partials = 0, scores = 0, hist = 0, total = kFlagBytes;
    int splits = 0;
};

Layout layout(const tsa::Dims& d, int k_max, int block, bool attn, bool dense, bool scores) {
    Layout L;
    size_t off = kFlagBytes;
    // The top-digit histograms must be zero when a decode step starts (its top-k
    // returns them to zero).  They sit at the same offset, right after the flag,
    // in every layout, so steps of any mode that share a workspace never write
    // over them with their split partials or scores.
    L.hist = off;
    off += a256((size_t)d.units() * tsa::kHistBins * sizeof(uint32_t));
    if (attn) {
        L.splits = tsa::attn_splits(d, k_max, block, dense);
        L.counters = off;
        off += a256((size_t)d.units() * sizeof(unsigned));
        L.partials = off;
        off += a256(tsa::attn_partials_floats(d, L.splits) * sizeof(float));
    }
    if (scores) {
        L.scores = off;
        off += a256((size_t)d.units() * tsa::rows_cap_of(d, block) * sizeof(float));
    }
    L.total = off;
    return L;
}

tsa_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
    if (ws == nullptr) return fail(TSA_ERR_WORKSPACE, "workspace pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(TSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (ws_bytes < need) return fail(TSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    return TSA_OK;
}

unsigned* flag_of(void* ws) { return static_cast<unsigned*>(ws); }

tsa_status check_kmax(int k_max) {
    if (k_max < 0) return fail(TSA_ERR_INVALID_ARG, "k_max must be >= 0 (got %d)", k_max);
    return TSA_OK;
}

}  // namespace

#define TSA_TRY(x)                       \
    do {                                 \
        tsa_status _st = (x);            \
        if (_st != TSA_OK) return _st;   \
    } while (0)

extern "C" {

size_t tsa_workspace_size(tsa_shape shape, int32_t k_max, int32_t block, int32_t mode) {
    tsa::Dims d;
    if (check_shape(shape, &d) != TSA_OK || check_block(block) != TSA_OK || check_kmax(k_max) != TSA_OK) return 0;
    switch (mode) {
        case TSA_FULL:  // k_max > 0: room for a layer that also emits its top-k
            return k_max > 0 ? layout(d, k_max, block, true, true, true).total : layout(d, 0, 1, true, true, false).total;
        case TSA_SELECT: return layout(d, k_max, block, true, false, true).total;
        case TSA_REUSE: return layout(d, k_max, block, true, false, false).total;
        default:
            fail(TSA_ERR_INVALID_ARG, "unknown mode %d", mode);
            return 0;
    }
}

tsa_status tsa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    TSA_TRY(check_ws(ws, ws_bytes, kFlagBytes));
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tsa_workspace_init");
    return TSA_OK;
}

tsa_status tsa_block_summarize(const void* K, const int32_t* seq_lens, tsa_shape shape,
                               int32_t block, float* Kmean, void* ws, size_t ws_bytes,
                               void* stream) {
    tsa::Dims d;
    TSA_TRY(check_shape(shape, &d));
    TSA_TRY(check_block(block));
    if (!K || !seq_lens || !Kmean) return fail(TSA_ERR_INVALID_ARG, "tsa_block_summarize: NULL pointer");
    if (!aligned16(K) || !aligned16(Kmean)) return fail(TSA_ERR_INVALID_ARG, "tsa_block_summarize: K and Kmean must be 16-byte aligned");
    TSA_TRY(check_ws(ws, ws_bytes, kFlagBytes));
    cudaError_t e = tsa::launch_block_summarize(K, seq_lens, d, block, Kmean, flag_of(ws),
                                                static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tsa_block_summarize");
    return TSA_OK;
}

tsa_status tsa_index_overlap(const int32_t* idx, int32_t n_layers, int32_t units, int32_t k_max,
                             int32_t* counts, double* M, void* ws, size_t ws_bytes, void* stream) {
    if (n_layers < 1 || n_layers > 1024)
        return fail(TSA_ERR_INVALID_ARG, "tsa_index_overlap: n_layers must be in [1, 1024] (got %d)", n_layers);
    if (units < 0 || k_max < 0)
        return fail(TSA_ERR_INVALID_ARG, "tsa_index_overlap: units and k_max must be >= 0 (got %d, %d)", units, k_max);
    if ((!idx && (size_t)units * k_max > 0) || (!counts && !M))
        return fail(TSA_ERR_INVALID_ARG, "tsa_index_overlap: NULL pointer (idx, or both counts and M)");
    TSA_TRY(check_ws(ws, ws_bytes, kFlagBytes));
    cudaError_t e = tsa::launch_index_overlap(idx, n_layers, units, k_max, counts, M, flag_of(ws),
                                              static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tsa_index_overlap");
    return TSA_OK;
}

// ---------------------------------------------------------------- sequence sharding

namespace {

tsa_status check_shards(int n_shards) {
    if (n_shards < 1 || n_shards > tsa::kMaxShards)
        return fail(TSA_ERR_INVALID_ARG, "n_shards must be in [1, %d] (got %d)", tsa::kMaxShards, n_shards);
    return TSA_OK;
}

// The four calls of a rank share one workspace, and none of them may write over
// the regions that must be zero when a call starts (the top-digit histograms and
// the split counters, right after the flag).  select and attend use
// [flag][histograms][counters][partials][scores][local rows]; the merge writes
// its scratch (candidate scores, candidate rows, counts, positions) from the end
// of the counters on, over space that select and attend use only inside a call,
// at offsets that do not depend on the shard's capacity.
struct ShardLayout {
    Layout front;  // select / attend
    size_t local, front_total;
    size_t pk_scores, pk_rows, n_cand, pos, merge_total;
    size_t total() const { return std::max(front_total, merge_total); }
};

ShardLayout shard_layout(const tsa::Dims& d, int k_max, int R) {
    ShardLayout S;
    S.front = layout(d, k_max, 1, true, false, true);
    S.local = S.front.total;
    S.front_total = S.local + a256((size_t)d.units() * k_max * 4);
    size_t off = S.front.partials;  // flag, histograms and counters come first in every layout
    const size_t wide = a256((size_t)d.units() * R * k_max * 4);
    S.pk_scores = off;
    off += wide;
    S.pk_rows = off;
    off += wide;
    S.n_cand = off;
    off += a256((size_t)d.B * 4);
    S.pos = off;
    off += a256((size_t)d.units() * k_max * 4);
    S.merge_total = off;
    return S;
}

}  // namespace

size_t tsa_shard_workspace_size(tsa_shape shard_shape, int32_t k_max, int32_t n_shards) {
    tsa::Dims d;
    if (check_shape(shard_shape, &d) != TSA_OK || check_kmax(k_max) != TSA_OK || check_shards(n_shards) != TSA_OK)
        return 0;
    return shard_layout(d, k_max, n_shards).total();
}

tsa_status tsa_shard_select(const void* Q, const void* K_shard, const int32_t* shard_lens, tsa_shape shard_shape,
                            const int32_t* k_per_seq, int32_t k_max, float scale, int32_t row0,
                            float* cand_scores, int32_t* cand_rows, void* ws, size_t ws_bytes, void* stream) {
    tsa::Dims d;
    TSA_TRY(check_shape(shard_shape, &d));
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_kmax(k_max));
    if (k_max == 0) return fail(TSA_ERR_INVALID_ARG, "tsa_shard_select: k_max must be > 0");
    if (row0 < 0 || (long long)row0 + d.Ncap > INT32_MAX)
        return fail(TSA_ERR_INVALID_ARG, "tsa_shard_select: row0 must be >= 0 and row0 + Ncap fit in int32");
    if (!Q || !K_shard || !shard_lens || !cand_scores || !cand_rows)
        return fail(TSA_ERR_INVALID_ARG, "tsa_shard_select: NULL pointer");
    if (!aligned16(Q) || !aligned16(K_shard)) return fail(TSA_ERR_INVALID_ARG, "tsa_shard_select: Q and K must be 16-byte aligned");
    int C, chunk;
    if (!tsa::topk_plan(d.Ncap, &C, &chunk))
        return fail(TSA_ERR_UNSUPPORTED, "tsa_shard_select: %d rows per unit exceed the top-k cluster capacity", d.Ncap);
    const Layout L = shard_layout(d, k_max, 1).front;
    TSA_TRY(check_ws(ws, ws_bytes, L.total));
    char* w = static_cast<char*>(ws);
    float* scores = reinterpret_cast<float*>(w + L.scores);
    uint32_t* hist = reinterpret_cast<uint32_t*>(w + L.hist);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = tsa::launch_score(Q, K_shard, shard_lens, d, 1, scale, scores, hist, flag_of(ws), st);
    if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_select (score)");
    e = tsa::launch_topk(scores, shard_lens, k_per_seq, k_max, d, 1, cand_rows, hist, flag_of(ws), st);
    if (e != cudaSuccess) {
        cudaMemsetAsync(hist, 0, (size_t)d.units() * tsa::kHistBins * sizeof(uint32_t), st);
        return cuda_fail(e, "tsa_shard_select (top-k)");
    }
    e = tsa::launch_shard_pack(scores, d.Ncap, d.units(), k_max, row0, cand_rows, cand_scores, flag_of(ws), st);
    if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_select (candidates)");
    return TSA_OK;
}

tsa_status tsa_shard_merge(const float* cand_scores, const int32_t* cand_rows, int32_t n_shards, tsa_shape shape,
                           const int32_t* k_per_seq, int32_t k_max, int32_t* idx, void* ws, size_t ws_bytes,
                           void* stream) {
    tsa::Dims d;
    TSA_TRY(check_shape(shape, &d));
    TSA_TRY(check_shards(n_shards));
    TSA_TRY(check_kmax(k_max));
    if (k_max == 0) return fail(TSA_ERR_INVALID_ARG, "tsa_shard_merge: k_max must be > 0");
    if (!cand_scores || !cand_rows || !idx) return fail(TSA_ERR_INVALID_ARG, "tsa_shard_merge: NULL pointer");
    const long long width = (long long)n_shards * k_max;
    int C, chunk;
    if (width > INT32_MAX || !tsa::topk_plan((int)width, &C, &chunk))
        return fail(TSA_ERR_UNSUPPORTED, "tsa_shard_merge: %lld candidates per unit exceed the top-k capacity", width);
    const ShardLayout S = shard_layout(d, k_max, n_shards);  // merge offsets do not depend on Ncap
    TSA_TRY(check_ws(ws, ws_bytes, S.merge_total));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (tsa::merge_topk_fits(n_shards, k_max)) {  // one kernel: the lists in one CTA's shared memory a unit
        const cudaError_t e = tsa::launch_merge_topk(cand_scores, cand_rows, n_shards, d.units(), d.Hkv, k_max,
                                                     k_per_seq, idx, flag_of(ws), st);
        if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_merge");
        return TSA_OK;
    }
    char* w = static_cast<char*>(ws);
    float* pk_scores = reinterpret_cast<float*>(w + S.pk_scores);
    int32_t* pk_rows = reinterpret_cast<int32_t*>(w + S.pk_rows);
    int32_t* n_cand = reinterpret_cast<int32_t*>(w + S.n_cand);
    int32_t* pos = reinterpret_cast<int32_t*>(w + S.pos);
    // the packing counts the candidates' first radix digit into the
    // histograms (zero here: every call that used them zeroed them), and the
    // top-k over the candidates starts from it
    uint32_t* hist = reinterpret_cast<uint32_t*>(w + S.front.hist);
    cudaError_t e = tsa::launch_merge_pack(cand_scores, cand_rows, n_shards, d.units(), d.Hkv, k_max, pk_scores,
                                           pk_rows, n_cand, hist, flag_of(ws), st);
    if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_merge (pack)");
    tsa::Dims dc = d;
    dc.Ncap = (int)width;  // the candidates are the rows of this top-k
    e = tsa::launch_topk(pk_scores, n_cand, k_per_seq, k_max, dc, 1, pos, hist, flag_of(ws), st);
    if (e != cudaSuccess) {
        cudaMemsetAsync(hist, 0, (size_t)d.units() * tsa::kHistBins * sizeof(uint32_t), st);
        return cuda_fail(e, "tsa_shard_merge (top-k)");
    }
    e = tsa::launch_merge_map(pos, pk_rows, d.units(), (int)width, k_max, idx, st);
    if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_merge (rows)");
    return TSA_OK;
}

tsa_status tsa_shard_attend(const void* Q, const void* K_shard, const void* V_shard, const int32_t* shard_lens,
                            tsa_shape shard_shape, const int32_t* idx, const int32_t* k_per_seq, int32_t k_max,
                            int32_t row0, float scale, float* O_part, float* lse_part, void* ws, size_t ws_bytes,
                            void* stream) {
    tsa::Dims d;
    TSA_TRY(check_shape(shard_shape, &d));
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_kmax(k_max));
    if (k_max == 0) return fail(TSA_ERR_INVALID_ARG, "tsa_shard_attend: k_max must be > 0");
    if (row0 < 0) return fail(TSA_ERR_INVALID_ARG, "tsa_shard_attend: row0 must be >= 0");
    if (!Q || !K_shard || !V_shard || !shard_lens || !idx || !O_part || !lse_part)
        return fail(TSA_ERR_INVALID_ARG, "tsa_shard_attend: NULL pointer");
    if (!aligned16(Q) || !aligned16(K_shard) || !aligned16(V_shard) || !aligned16(O_part))
        return fail(TSA_ERR_INVALID_ARG, "tsa_shard_attend: Q, K, V and O_part must be 16-byte aligned");
    const ShardLayout S = shard_layout(d, k_max, 1);
    const Layout& L = S.front;
    TSA_TRY(check_ws(ws, ws_bytes, S.front_total));
    char* w = static_cast<char*>(ws);
    int32_t* local = reinterpret_cast<int32_t*>(w + S.local);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = tsa::launch_localize(idx, d.units(), k_max, row0, d.Ncap, local, st);
    if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_attend (local rows)");
    e = tsa::launch_attn(Q, K_shard, V_shard, shard_lens, local, k_per_seq, k_max, 1, d, scale, L.splits,
                         reinterpret_cast<float*>(w + L.partials), reinterpret_cast<unsigned*>(w + L.counters), O_part,
                         flag_of(ws), st, 0, nullptr, false, lse_part);
    if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_attend (attention)");
    return TSA_OK;
}

tsa_status tsa_shard_combine(const float* O_parts, const float* lse_parts, int32_t n_shards, tsa_shape shape,
                             float* O, void* stream) {
    tsa::Dims d;
    TSA_TRY(check_shape(shape, &d));
    TSA_TRY(check_shards(n_shards));
    if (!O_parts || !lse_parts || !O) return fail(TSA_ERR_INVALID_ARG, "tsa_shard_combine: NULL pointer");
    if (!aligned16(O_parts) || !aligned16(O))
        return fail(TSA_ERR_INVALID_ARG, "tsa_shard_combine: O_parts and O must be 16-byte aligned");
    cudaError_t e = tsa::launch_shard_combine(O_parts, lse_parts, n_shards, d.B * d.Hq, O,
                                              static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tsa_shard_combine");
    return TSA_OK;
}

tsa_status sparse_decode_score(const void* Q, const void* keys, const int32_t* seq_lens,
                               tsa_shape shape, int32_t block, float scale, float* scores,
                               void* ws, size_t ws_bytes, void* stream) {
    tsa::Dims d;
    TSA_TRY(check_shape(shape, &d));
    TSA_TRY(check_block(block));
    TSA_TRY(check_scale(scale));
    if (!Q || !keys || !seq_lens || !scores) return fail(TSA_ERR_INVALID_ARG, "sparse_decode_score: NULL pointer");
    if (!aligned16(Q) || !aligned16(keys)) return fail(TSA_ERR_INVALID_ARG, "sparse_decode_score: Q and keys must be 16-byte aligned");
    TSA_TRY(check_ws(ws, ws_bytes, kFlagBytes));
    cudaError_t e = tsa::launch_score(Q, keys, seq_lens, d, block, scale, scores, nullptr, flag_of(ws),
                                      static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "sparse_decode_score");
    return TSA_OK;
}

tsa_status topk_select(const float* scores, const int32_t* seq_lens, const int32_t* k_per_seq,
                       int32_t k_max, tsa_shape shape, int32_t block, int32_t* idx, void* ws,
                       size_t ws_bytes, void* stream) {
    tsa::Dims d;
    TSA_TRY(check_shape(shape, &d));
    TSA_TRY(check_block(block));
    TSA_TRY(check_kmax(k_max));
    if (!scores || !seq_lens || !idx) return fail(TSA_ERR_INVALID_ARG, "topk_select: NULL pointer");
    int C, chunk;
    if (!tsa::topk_plan(tsa::rows_cap_of(d, block), &C, &chunk))
        return fail(TSA_ERR_UNSUPPORTED, "topk_select: %d rows per unit exceed the cluster capacity", tsa::rows_cap_of(d, block));
    TSA_TRY(check_ws(ws, ws_bytes, kFlagBytes));
    cudaError_t e = tsa::launch_topk(scores, seq_lens, k_per_seq, k_max, d, block, idx, nullptr,
                                     flag_of(ws), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "topk_select");
    return TSA_OK;
}

namespace {

// K and V of an offloaded cache: page-locked host memory that the device reads
// at the same address (cudaHostAlloc, or cudaHostRegister'd and mapped).  Any
// other host pointer (pageable memory) would fault the kernel, so it is refused.
tsa_status check_host_kv(const void* K, const void* V) {
    const void* ptrs[2] = {K, V};
    for (const void* p : ptrs) {
        cudaPointerAttributes at;
        cudaError_t e = cudaPointerGetAttributes(&at, p);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, "tsa_decode_step (K/V pointer query)");
        }
        if (at.type != cudaMemoryTypeHost || at.devicePointer != p)
            return fail(TSA_ERR_INVALID_ARG,
                        "tsa_decode_step: with TSA_KV_HOST, K and V must be page-locked host memory mapped for "
                        "the device at the same address (cudaHostAlloc, or cudaHostRegister with mapping)");
    }
    return TSA_OK;
}

tsa_status attn_stage(const void* Q, const void* K, const void* V, const int32_t* seq_lens, const int32_t* idx,
                      const int32_t* k_per_seq, int32_t k_max, int32_t block, tsa_shape shape, float scale, float* O,
                      void* ws, size_t ws_bytes, void* stream, bool host_kv, int early);

}  // namespace

tsa_status sparse_decode_attn(const void* Q, const void* K, const void* V,
                              const int32_t* seq_lens, const int32_t* idx,
                              const int32_t* k_per_seq, int32_t k_max, int32_t block,
                              tsa_shape shape, float scale, float* O, void* ws, size_t ws_bytes,
                              void* stream) {
    return attn_stage(Q, K, V, seq_lens, idx, k_per_seq, k_max, block, shape, scale, O, ws, ws_bytes, stream,
                      false, 0);
}

namespace {

tsa_status attn_stage(const void* Q, const void* K, const void* V, const int32_t* seq_lens, const int32_t* idx,
                      const int32_t* k_per_seq, int32_t k_max, int32_t block, tsa_shape shape, float scale, float* O,
                      void* ws, size_t ws_bytes, void* stream, bool host_kv, int early) {
    tsa::Dims d;
    TSA_TRY(check_shape(shape, &d));
    TSA_TRY(check_block(block));
    TSA_TRY(check_scale(scale));
    TSA_TRY(check_kmax(k_max));
    if (!Q || !K || !V || !seq_lens || !O) return fail(TSA_ERR_INVALID_ARG, "sparse_decode_attn: NULL pointer");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return fail(TSA_ERR_INVALID_ARG, "sparse_decode_attn: Q, K, V and O must be 16-byte aligned");
    const bool dense = idx == nullptr;
    if (!dense && k_max == 0) return fail(TSA_ERR_INVALID_ARG, "sparse_decode_attn: k_max must be > 0 with an index list");
    const Layout L = layout(d, dense ? 0 : k_max, dense ? 1 : block, true, dense, false);
    TSA_TRY(check_ws(ws, ws_bytes, L.total));
    char* w = static_cast<char*>(ws);
    if (host_kv) TSA_TRY(check_host_kv(K, V));
    cudaError_t e = tsa::launch_attn(Q, K, V, seq_lens, idx, k_per_seq, k_max, dense ? 1 : block, d,
                                     scale, L.splits, reinterpret_cast<float*>(w + L.partials),
                                     reinterpret_cast<unsigned*>(w + L.counters), O, flag_of(ws),
                                     static_cast<cudaStream_t>(stream), early, nullptr, host_kv);
    if (e != cudaSuccess) return cuda_fail(e, "sparse_decode_attn");
    return TSA_OK;
}

}  // namespace

tsa_status tsa_decode_step(const tsa_step_args* a, void* stream) {
    if (!a) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: NULL args");
    tsa::Dims d;
    TSA_TRY(check_shape(a->shape, &d));
    if (a->flags & ~(uint32_t)(TSA_KV_HOST | TSA_EARLY_INPUTS))
        return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: unknown flags 0x%x", a->flags);
    const bool host_kv = (a->flags & TSA_KV_HOST) != 0;
    // the caller's promise (TSA_EARLY_INPUTS): the first kernel of the step may
    // read lens, k's, K, V and idx_in before the kernel before it has finished
    const bool early_in = (a->flags & TSA_EARLY_INPUTS) != 0;
    if (host_kv && a->block == 1 && (a->mode == TSA_SELECT || (a->mode == TSA_FULL && a->idx_out)))
        return fail(TSA_ERR_UNSUPPORTED,
                    "tsa_decode_step: with TSA_KV_HOST a layer that selects must score block means (block > 1); "
                    "token-mode scoring streams all of K");
    switch (a->mode) {
        case TSA_FULL: {
            if (!a->idx_out)
                return attn_stage(a->Q, a->K, a->V, a->seq_lens, nullptr, nullptr, 0, 1, a->shape, a->scale, a->O,
                                  a->ws, a->ws_bytes, stream, host_kv, early_in ? 2 : 0);
            // A full layer that also hands its top-k on (HyLRA: a sensitive layer's
            // extracted indices pass to the tolerant layers after it).  Token mode:
            // the full attention writes each row's score as it forms S (no second
            // read of K), then the top-k.  Block mode: the block means are scored
            // as in a SELECT step.
            TSA_TRY(check_block(a->block));
            TSA_TRY(check_scale(a->scale));
            TSA_TRY(check_kmax(a->k_max));
            if (a->k_max == 0) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: a TSA_FULL layer with idx_out needs k_max > 0");
            if (a->block > 1 && !a->Kmean) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: block mode needs Kmean");
            if (!a->Q || !a->K || !a->V || !a->seq_lens || !a->O) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: NULL pointer");
            if (!aligned16(a->Q) || !aligned16(a->K) || !aligned16(a->V) || !aligned16(a->O) ||
                (a->block > 1 && !aligned16(a->Kmean)))
                return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: Q, K, V, Kmean and O must be 16-byte aligned");
            int C, chunk;
            if (!tsa::topk_plan(tsa::rows_cap_of(d, a->block), &C, &chunk))
                return fail(TSA_ERR_UNSUPPORTED, "tsa_decode_step: %d rows per unit exceed the top-k cluster capacity",
                            tsa::rows_cap_of(d, a->block));
            const Layout L = layout(d, a->k_max, a->block, true, true, true);
            TSA_TRY(check_ws(a->ws, a->ws_bytes, L.total));
            if (host_kv) TSA_TRY(check_host_kv(a->K, a->V));
            char* w = static_cast<char*>(a->ws);
            float* scores = reinterpret_cast<float*>(w + L.scores);
            uint32_t* hist = reinterpret_cast<uint32_t*>(w + L.hist);
            float* partials = reinterpret_cast<float*>(w + L.partials);
            unsigned* counters = reinterpret_cast<unsigned*>(w + L.counters);
            cudaStream_t st = static_cast<cudaStream_t>(stream);
            cudaError_t e;
            if (a->block == 1) {
                // the attention also counts the scores' first radix digit, so the
                // top-k that follows starts from that histogram (and zeroes it)
                e = tsa::launch_attn(a->Q, a->K, a->V, a->seq_lens, nullptr, nullptr, 0, 1, d, a->scale, L.splits,
                                     partials, counters, a->O, flag_of(a->ws), st, early_in ? 2 : 0, scores, false,
                                     nullptr, hist);
                if (e != cudaSuccess) return cuda_fail(e, "tsa_decode_step (full attention)");
                e = tsa::launch_topk(scores, a->seq_lens, a->k_per_seq, a->k_max, d, 1, a->idx_out, hist,
                                     flag_of(a->ws), st);
                if (e != cudaSuccess) {
                    cudaMemsetAsync(hist, 0, (size_t)d.units() * tsa::kHistBins * sizeof(uint32_t), st);
                    return cuda_fail(e, "tsa_decode_step (top-k)");
                }
                return TSA_OK;
            }
            e = tsa::launch_score(a->Q, a->Kmean, a->seq_lens, d, a->block, a->scale, scores, hist, flag_of(a->ws), st);
            if (e != cudaSuccess) return cuda_fail(e, "tsa_decode_step (score)");
            e = tsa::launch_topk(scores, a->seq_lens, a->k_per_seq, a->k_max, d, a->block, a->idx_out, hist,
                                 flag_of(a->ws), st);
            if (e != cudaSuccess) {
                cudaMemsetAsync(hist, 0, (size_t)d.units() * tsa::kHistBins * sizeof(uint32_t), st);
                return cuda_fail(e, "tsa_decode_step (top-k)");
            }
            e = tsa::launch_attn(a->Q, a->K, a->V, a->seq_lens, nullptr, nullptr, 0, 1, d, a->scale, L.splits,
                                 partials, counters, a->O, flag_of(a->ws), st, 0, nullptr, host_kv);
            if (e != cudaSuccess) return cuda_fail(e, "tsa_decode_step (full attention)");
            return TSA_OK;
        }
        case TSA_REUSE:
            if (!a->idx_in) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: TSA_REUSE needs idx_in");
            return attn_stage(a->Q, a->K, a->V, a->seq_lens, a->idx_in, a->k_per_seq, a->k_max, a->block, a->shape,
                              a->scale, a->O, a->ws, a->ws_bytes, stream, host_kv, early_in ? 2 : 0);
        case TSA_SELECT: {
            TSA_TRY(check_block(a->block));
            TSA_TRY(check_scale(a->scale));
            TSA_TRY(check_kmax(a->k_max));
            if (a->k_max == 0) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: TSA_SELECT needs k_max > 0");
            if (!a->idx_out) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: TSA_SELECT needs idx_out");
            if (a->block > 1 && !a->Kmean) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: block mode needs Kmean");
            if (!a->Q || !a->K || !a->V || !a->seq_lens || !a->O) return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: NULL pointer");
            if (!aligned16(a->Q) || !aligned16(a->K) || !aligned16(a->V) || !aligned16(a->O) ||
                (a->block > 1 && !aligned16(a->Kmean)))
                return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: Q, K, V, Kmean and O must be 16-byte aligned");
            int C, chunk;
            if (!tsa::topk_plan(tsa::rows_cap_of(d, a->block), &C, &chunk))
                return fail(TSA_ERR_UNSUPPORTED, "tsa_decode_step: %d rows per unit exceed the top-k cluster capacity",
                            tsa::rows_cap_of(d, a->block));
            const Layout L = layout(d, a->k_max, a->block, true, false, true);
            TSA_TRY(check_ws(a->ws, a->ws_bytes, L.total));
            if (host_kv) TSA_TRY(check_host_kv(a->K, a->V));
            char* w = static_cast<char*>(a->ws);
            float* scores = reinterpret_cast<float*>(w + L.scores);
            // the scorer also histograms the top digit of its keys; the top-k
            // starts from that histogram and zeroes it for the next step
            uint32_t* hist = reinterpret_cast<uint32_t*>(w + L.hist);
            const void* keys = a->block == 1 ? a->K : static_cast<const void*>(a->Kmean);
            cudaStream_t st = static_cast<cudaStream_t>(stream);
            cudaError_t e = tsa::launch_score(a->Q, keys, a->seq_lens, d, a->block, a->scale, scores, hist,
                                              flag_of(a->ws), st, early_in);
            if (e != cudaSuccess) return cuda_fail(e, "tsa_decode_step (score)");
            e = tsa::launch_topk(scores, a->seq_lens, a->k_per_seq, a->k_max, d, a->block, a->idx_out, hist,
                                 flag_of(a->ws), st);
            if (e != cudaSuccess) {
                // leave no partial histogram behind for the next step (best effort)
                cudaMemsetAsync(hist, 0, (size_t)d.units() * tsa::kHistBins * sizeof(uint32_t), st);
                return cuda_fail(e, "tsa_decode_step (top-k)");
            }
            // the attention follows this step's own top-k, which wrote only the
            // indices: it may read the lengths, k's and Q before waiting on it
            e = tsa::launch_attn(a->Q, a->K, a->V, a->seq_lens, a->idx_out, a->k_per_seq, a->k_max, a->block, d,
                                 a->scale, L.splits, reinterpret_cast<float*>(w + L.partials),
                                 reinterpret_cast<unsigned*>(w + L.counters), a->O, flag_of(a->ws), st, 1,
                                 nullptr, host_kv);
            if (e != cudaSuccess) return cuda_fail(e, "tsa_decode_step (attention)");
            return TSA_OK;
        }
        default:
            return fail(TSA_ERR_INVALID_ARG, "tsa_decode_step: unknown mode %d", a->mode);
    }
}

tsa_status tsa_check_device_status(void* ws, void* stream) {
    if (!ws) return fail(TSA_ERR_INVALID_ARG, "tsa_check_device_status: NULL workspace");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof h, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof h, st);
    if (e != cudaSuccess) return cuda_fail(e, "tsa_check_device_status");
    if (h & tsa::kFlagTimeoutBit) return fail(TSA_ERR_DEVICE_TIMEOUT, "a bounded device-side wait gave up");
    if (h & tsa::kFlagBoundsBit) return fail(TSA_ERR_DEVICE_BOUNDS, "device saw a length, k or index out of range");
    return TSA_OK;
}

const char* tsa_last_error_string(void) { return g_err; }

uint64_t tsa_launch_count(void) { return tsa::g_launches.load(std::memory_order_relaxed); }

tsa_status tsa_hbm_copy(const void* src, void* dst, size_t bytes, void* stream) {
    if (!src || !dst) return fail(TSA_ERR_INVALID_ARG, "tsa_hbm_copy: NULL pointer");
    if (!aligned16(src) || !aligned16(dst) || bytes % 16 != 0)
        return fail(TSA_ERR_INVALID_ARG, "tsa_hbm_copy: pointers and size must be multiples of 16 bytes");
    cudaError_t e = tsa::launch_copy(src, dst, bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tsa_hbm_copy");
    return TSA_OK;
}

tsa_status tsa_hbm_read(const void* src, size_t bytes, void* ws, size_t ws_bytes, void* stream) {
    if (!src) return fail(TSA_ERR_INVALID_ARG, "tsa_hbm_read: NULL pointer");
    if (!aligned16(src) || bytes % 16 != 0)
        return fail(TSA_ERR_INVALID_ARG, "tsa_hbm_read: pointer and size must be multiples of 16 bytes");
    TSA_TRY(check_ws(ws, ws_bytes, kFlagBytes));
    // the fold's landing word: inside the flag block, past the flag itself
    unsigned* sink = flag_of(ws) + 1;
    cudaError_t e = tsa::launch_read(src, bytes, sink, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tsa_hbm_read");
    return TSA_OK;
}

tsa_status tsa_hbm_gather(const void* base, size_t base_bytes, const int32_t* rows, int32_t nrows, void* ws,
                          size_t ws_bytes, void* stream) {
    if (!base || (!rows && nrows > 0)) return fail(TSA_ERR_INVALID_ARG, "tsa_hbm_gather: NULL pointer");
    if (!aligned16(base) || base_bytes % 256 != 0)
        return fail(TSA_ERR_INVALID_ARG, "tsa_hbm_gather: base must be 16-byte aligned and a whole number of 256-byte rows");
    if (nrows < 0) return fail(TSA_ERR_INVALID_ARG, "tsa_hbm_gather: nrows must be >= 0");
    TSA_TRY(check_ws(ws, ws_bytes, kFlagBytes));
    cudaError_t e = tsa::launch_gather(base, base_bytes, rows, nrows, flag_of(ws), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "tsa_hbm_gather");
    return TSA_OK;
}

}  // extern "C"
