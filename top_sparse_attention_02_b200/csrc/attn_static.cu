// attn_static.cu -- sparse_decode_attn_noalloc: the attention stage with its
// scratch (split counters and split partials) in a fixed device array that
// the library owns, for callers that cannot hand the library a workspace.
//
// Some callers cannot allocate device memory for a workspace: a plugin host
// that gives an operator only its input and output buffers, a runtime whose
// device memory all belongs to another allocator, or a steady-state serving
// loop that must not call cudaMalloc/cudaFree (cudaFree synchronises the whole
// device, and cudaMalloc may block).  This entry point takes the same inputs
// and outputs as sparse_decode_attn and uses `g_attn_scratch` below instead of
// `ws`.  It calls no cudaMalloc, cudaFree or allocating library routine.
#include <cmath>
#include <cstdio>

#include "common.cuh"
#include "launch.h"
#include "tsa.h"

namespace {

constexpr size_t kScratchBytes = (size_t)8 << 20;  // 8 MiB, held by every GPU that loads the library
constexpr size_t kFlagBytes = 256;

// File-scope device scratch.  In host code this name is only a stand-in for the
// device array, never a device address: the address comes from
// cudaGetSymbolAddress, on every call, with the calling device current.
static __device__ __align__(256) unsigned char g_attn_scratch[kScratchBytes];

tsa_status bad(tsa_status st, const char* msg) {
    tsa::set_error_message(msg);  // read back with tsa_last_error_string()
    return st;
}

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

extern "C" {

tsa_status sparse_decode_attn_noalloc(const void* Q, const void* K, const void* V,
                                      const int32_t* seq_lens, const int32_t* idx,
                                      const int32_t* k_per_seq, int32_t k_max, int32_t block,
                                      tsa_shape shape, float scale, float* O, void* stream) {
    // ---- the same argument rules as sparse_decode_attn
    if (shape.B < 0 || shape.Hq <= 0 || shape.Hkv <= 0 || shape.Ncap < 0 || shape.Hq % shape.Hkv != 0)
        return bad(TSA_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: bad shape");
    if (shape.d != tsa::kDHead) return bad(TSA_ERR_UNSUPPORTED, "sparse_decode_attn_noalloc: d must be 128");
    const int G = shape.Hq / shape.Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return bad(TSA_ERR_UNSUPPORTED, "sparse_decode_attn_noalloc: Hq/Hkv must be 1, 2, 4 or 8");
    if ((long long)shape.B * shape.Hkv > 65535)
        return bad(TSA_ERR_UNSUPPORTED, "sparse_decode_attn_noalloc: B*Hkv above 65535");
    if (block < 1 || block > 4096) return bad(TSA_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: block must be in [1, 4096]");
    if (!std::isfinite(scale) || !(scale > 0.f)) return bad(TSA_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: scale must be finite and > 0");
    if (k_max < 0 || (idx != nullptr && k_max == 0)) return bad(TSA_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: bad k_max");
    if (!Q || !K || !V || !seq_lens || !O) return bad(TSA_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: NULL pointer");
    if (((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) |
          reinterpret_cast<uintptr_t>(O)) & 15u) != 0)
        return bad(TSA_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: Q, K, V and O must be 16-byte aligned");

    tsa::Dims d{shape.B, shape.Hq, shape.Hkv, shape.Ncap, G};
    const bool dense = idx == nullptr;
    const int blk = dense ? 1 : block;
    const int splits = tsa::attn_splits(d, dense ? 0 : k_max, blk, dense);
    const size_t counters = kFlagBytes;
    const size_t partials = counters + a256((size_t)d.units() * sizeof(unsigned));
    const size_t need = partials + a256(tsa::attn_partials_floats(d, splits) * sizeof(float));
    char msg[256];
    if (need > kScratchBytes) {
        snprintf(msg, sizeof msg,
                 "sparse_decode_attn_noalloc: this shape needs %zu bytes of scratch; the fixed array "
                 "holds %zu (use sparse_decode_attn with a workspace)", need, kScratchBytes);
        return bad(TSA_ERR_WORKSPACE, msg);
    }

    // ---- the array's device address on the current device.  Looked up on
    // every call (it allocates nothing and is cheap), so that it is never stale:
    // after cudaDeviceReset, or with another primary context, the library's
    // module is loaded again and the array may sit elsewhere.  The first call
    // on a device loads the module (with lazy loading) and so commits the array.
    void* base = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&base, g_attn_scratch);
    if (e != cudaSuccess || base == nullptr) {
        snprintf(msg, sizeof msg, "sparse_decode_attn_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        return bad(TSA_ERR_CUDA, msg);
    }
    char* s = static_cast<char*>(base);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the device flag and the
    // split counters must start at zero
    e = cudaMemsetAsync(s, 0, partials, st);
    if (e != cudaSuccess) return bad(TSA_ERR_CUDA, "sparse_decode_attn_noalloc: clearing the scratch failed");
    e = tsa::launch_attn(Q, K, V, seq_lens, idx, k_per_seq, k_max, blk, d, scale, splits,
                         reinterpret_cast<float*>(s + partials), reinterpret_cast<unsigned*>(s + counters),
                         O, reinterpret_cast<unsigned*>(s), st);
    if (e != cudaSuccess) {
        snprintf(msg, sizeof msg, "sparse_decode_attn_noalloc: %s", cudaGetErrorString(e));
        return bad(TSA_ERR_CUDA, msg);
    }
    return TSA_OK;
}

}  // extern "C"
