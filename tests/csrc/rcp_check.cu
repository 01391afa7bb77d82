// Exhaustive device check of rcp2_rn_mid and its one-lane form rcp_rn_mid
// (mxq_device.cuh): for every fp32 significand at every exponent of
// [2^-60, 2^60), both signs, the refined reciprocals must equal __frcp_rn
// (CUDA's correctly rounded reciprocal) bit for bit.  Prints "mismatches N first 0x........" and
// exits 0 when the run itself succeeded (the count is judged by the test).
#include <stdio.h>
#include "mxq_device.cuh"

__global__ void rcp_check_kernel(unsigned long long *bad, unsigned int *first)
{
    const unsigned int n = 1u << 23;
    for (unsigned int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        for (unsigned int e = 127 - 60; e < 127 + 60; ++e) {
            const float d = __uint_as_float((e << 23) | i);
            const float want = __frcp_rn(d);
            const float2 got = mxq::rcp2_rn_mid(make_float2(d, -d));
            const float one = mxq::rcp_rn_mid(e & 1u ? -d : d);
            if (__float_as_uint(got.x) != __float_as_uint(want) ||
                __float_as_uint(got.y) != (__float_as_uint(want) ^ 0x80000000u) ||
                __float_as_uint(one) != (__float_as_uint(want) ^ (e & 1u ? 0x80000000u : 0u))) {
                atomicAdd(bad, 1ull);
                atomicMin(first, (e << 23) | i);
            }
        }
    }
}

int main()
{
    unsigned long long *bad = nullptr, h_bad = 0;
    unsigned int *first = nullptr, h_first = 0;
    if (cudaMalloc(&bad, sizeof(*bad)) != cudaSuccess || cudaMalloc(&first, sizeof(*first)) != cudaSuccess) {
        printf("allocation failed\n");
        return 1;
    }
    cudaMemset(bad, 0, sizeof(*bad));
    cudaMemset(first, 0xFF, sizeof(*first));
    rcp_check_kernel<<<148 * 4, 256>>>(bad, first);
    cudaError_t err = cudaDeviceSynchronize();
    if (err == cudaSuccess)
        err = cudaMemcpy(&h_bad, bad, sizeof(h_bad), cudaMemcpyDeviceToHost);
    if (err == cudaSuccess)
        err = cudaMemcpy(&h_first, first, sizeof(h_first), cudaMemcpyDeviceToHost);
    if (err != cudaSuccess) {
        printf("CUDA error %s\n", cudaGetErrorString(err));
        return 1;
    }
    printf("mismatches %llu first 0x%08x\n", h_bad, h_first);
    return 0;
}
