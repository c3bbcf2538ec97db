// Weight repacking at load time: a tiled transpose so that every channel's
// gate / up / LoPA-B weights become one contiguous row (channel-major).
#include "common.cuh"

namespace sffn {

template <class T>
__global__ void k_transpose(const T* __restrict__ src, T* __restrict__ dst, int rows, int cols) {
    __shared__ T tile[32][33];
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < rows && c < cols) tile[i][threadIdx.x] = src[(size_t)r * cols + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (c < cols && r < rows) dst[(size_t)c * rows + r] = tile[threadIdx.x][i];
    }
}

// dst (cols x rows) = transpose of src (rows x cols), both row-major.
cudaError_t launch_transpose(int wdtype, const void* src, void* dst, int rows, int cols, cudaStream_t s) {
    if (rows <= 0 || cols <= 0) return cudaSuccess;
    if ((rows + 31) / 32 > 65535) return cudaErrorInvalidValue;
    const dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
    if (wdtype == 0)
        k_transpose<bf16><<<grid, block, 0, s>>>(static_cast<const bf16*>(src), static_cast<bf16*>(dst), rows, cols);
    else
        k_transpose<float><<<grid, block, 0, s>>>(static_cast<const float*>(src), static_cast<float*>(dst), rows, cols);
    return cudaGetLastError();
}

}  // namespace sffn
