// copy.cu -- HBM roofline probes.
//  - copy: a plain 16-byte-vector device-to-device copy over a grid sized to the
//    SM count; its bandwidth (read + write bytes / time) is the streaming peak
//    the scan kernels are compared against in the same run.
//  - read: the same loads with no stores; its bandwidth is the ceiling
//    of a read-only stream (the scorer's scan of K reads and hardly writes),
//    which a copy (half of its bytes written) understates;
//  - gather: 256-byte rows at given row numbers, fetched by TMA bulk copies into
//    shared memory and dropped; its bandwidth is the random-row ceiling the
//    attention stage (which gathers the selected K/V rows) is compared against.
#include "common.cuh"
#include "launch.h"

namespace tsa {

__global__ void __launch_bounds__(256) copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                   size_t n16) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = ld_stream(src + i), b = ld_stream(src + i + stride);
        const uint4 c = ld_stream(src + i + 2 * stride), d = ld_stream(src + i + 3 * stride);
        dst[i] = a;
        dst[i + stride] = b;
        dst[i + 2 * stride] = c;
        dst[i + 3 * stride] = d;
    }
    for (; i < n16; i += stride) dst[i] = ld_stream(src + i);
}

// the loaded words are folded into one value, stored only when it equals a
// value it cannot have for the probe's buffer of repeated bytes (so no load is
// removed and nothing is written)
__global__ void __launch_bounds__(256) read_kernel(const uint4* __restrict__ src, size_t n16,
                                                   unsigned* __restrict__ sink) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    unsigned acc = 0u;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = ld_stream(src + i), b = ld_stream(src + i + stride);
        const uint4 c = ld_stream(src + i + 2 * stride), d = ld_stream(src + i + 3 * stride);
        acc += (a.x ^ a.w) + (b.x ^ b.w) + (c.x ^ c.w) + (d.x ^ d.w);
    }
    for (; i < n16; i += stride) acc += ld_stream(src + i).y;
    if (acc == 0x9e3779b9u) *sink = acc;
}

constexpr int kGatherRowsPerCta = 256;  // a 64 KB shared-memory window per CTA
constexpr long kGatherSpins = 1L << 22;

__global__ void __launch_bounds__(128) gather_kernel(const unsigned char* __restrict__ base, size_t nrows_base,
                                                     const int32_t* __restrict__ rows, int nrows,
                                                     unsigned* __restrict__ flag) {
    extern __shared__ __align__(128) unsigned char gsm[];
    __shared__ __align__(8) uint64_t bar;
    const unsigned bar_a = (unsigned)__cvta_generic_to_shared(&bar);
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar_a), "r"(128) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    const int r0 = blockIdx.x * kGatherRowsPerCta;
    const int r1 = min(r0 + kGatherRowsPerCta, nrows);
    unsigned bytes = 0;
    for (int j = r0 + threadIdx.x; j < r1; j += 128) {
        const int32_t r = rows[j];
        if (r >= 0 && (size_t)r < nrows_base) bytes += 256;
    }
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(bar_a),
                 "r"(bytes)
                 : "memory");
    for (int j = r0 + threadIdx.x; j < r1; j += 128) {
        const int32_t r = rows[j];
        if (r < 0 || (size_t)r >= nrows_base) {
            atomicOr(flag, kFlagBounds);
            continue;
        }
        const unsigned dst = (unsigned)__cvta_generic_to_shared(gsm + (j - r0) * 256);
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 256, [%2];\n" ::"r"(
                         dst),
                     "l"(base + (size_t)r * 256), "r"(bar_a)
                     : "memory");
    }
    for (long i = 0; i < kGatherSpins; ++i) {
        unsigned done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(bar_a)
            : "memory");
        if (done) return;
    }
    atomicOr(flag, kFlagTimeout);
}

cudaError_t launch_gather(const void* base, size_t base_bytes, const int32_t* rows, int nrows, unsigned* flag,
                          cudaStream_t st) {
    if (nrows <= 0) return cudaSuccess;
    static int configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGatherRowsPerCta * 256);
        if (e != cudaSuccess) return e;
        configured[dev] = 1;
    }
    gather_kernel<<<ceil_div(nrows, kGatherRowsPerCta), 128, kGatherRowsPerCta * 256, st>>>(
        static_cast<const unsigned char*>(base), base_bytes / 256, rows, nrows, flag);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_read(const void* src, size_t bytes, unsigned* sink, cudaStream_t st) {
    if (bytes == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // 16 CTAs an SM (more requests in flight than the copy's 8; measured fastest)
    read_kernel<<<sms * 16, 256, 0, st>>>(static_cast<const uint4*>(src), bytes / 16, sink);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t st) {
    if (bytes == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    copy_kernel<<<sms * 8, 256, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                         bytes / 16);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tsa
