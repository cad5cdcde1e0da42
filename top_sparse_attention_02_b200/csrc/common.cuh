// common.cuh -- device helpers shared by the libtsa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace tsa {

constexpr int kD = kDHead;
constexpr unsigned kFlagBounds = kFlagBoundsBit;
constexpr unsigned kFlagTimeout = kFlagTimeoutBit;
constexpr float kLog2e = 1.4426950408889634f;

// 16-byte streaming load: read-only path, no L1 allocation (each K/V byte is used once).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

// bf16 pair in one 32-bit word -> two fp32 (exact: bf16 is the top half of fp32).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4& r, float (&f)[8]) {
    f[0] = bf_lo(r.x); f[1] = bf_hi(r.x);
    f[2] = bf_lo(r.y); f[3] = bf_hi(r.y);
    f[4] = bf_lo(r.z); f[5] = bf_hi(r.z);
    f[6] = bf_lo(r.w); f[7] = bf_hi(r.w);
}

// fp32 score -> unsigned key with the same order (larger float -> larger key).
// -0 is folded onto +0 so that the two compare equal, as the reals do.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Reduce 16 values held by each lane of a 16-lane half-warp so that, afterwards,
// lane c of the half holds in v[0] the sum over the half of value index c
// (a reduce-scatter by halving: 8+4+2+1 shuffles instead of 16*4).
__device__ __forceinline__ void halfwarp_reduce_scatter16(float (&v)[16], int c) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = c & 8;
        float send = up ? v[i] : v[i + 8];
        float keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = c & 4;
        float send = up ? v[i] : v[i + 4];
        float keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = c & 2;
        float send = up ? v[i] : v[i + 2];
        float keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    {
        const bool up = c & 1;
        float send = up ? v[0] : v[1];
        float keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
}

// Programmatic dependent launch: the kernels of a decode step are launched so
// that the next one may start (launch, set-up) while this one finishes.  Every
// kernel waits for its predecessor before touching global memory, which keeps
// the stream's order for data; and lets its successor launch once all of its
// CTAs are running.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// A hint that brings the 128-byte line holding p into L2; no data returns, so
// it may be issued before waiting on the kernel that writes p (L2 is where that
// kernel's writes land: the read after the wait sees them).
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p)); }

__device__ __forceinline__ int clamp_len(int len, int Ncap, unsigned* flag) {
    if (len < 0 || len > Ncap) {
        atomicOr(flag, kFlagBounds);
        len = len < 0 ? 0 : Ncap;
    }
    return len;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace tsa
