// copy.cu -- HBM roofline probe: a plain 16-byte-vector device-to-device copy
// over a grid sized to the SM count.  Its bandwidth (read + write bytes / time)
// is the denominator the decode kernels are compared against in the same run.
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
