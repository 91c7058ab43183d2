// Test helper: evaluates the library's FMA-pipe exp2 (exp2_poly2) and the MUFU ex2 on an
// array of inputs so the test can compare both with 2^x in float64.
#include <cstdint>
#include "ptx_sm100.cuh"

__global__ void probe(const float *x, float *poly, float *mufu, int n)
{
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        const float2 r = fa::ptx::exp2_poly2(make_float2(x[i], x[i + 1]));
        poly[i] = r.x;
        poly[i + 1] = r.y;
        mufu[i] = fa::ptx::ex2(x[i]);
        mufu[i + 1] = fa::ptx::ex2(x[i + 1]);
    }
}

extern "C" int exp2_probe(const float *x, float *poly, float *mufu, int n)
{
    if (n <= 0 || (n & 1)) return 1;
    const int pairs = n / 2;
    probe<<<(pairs + 255) / 256, 256>>>(x, poly, mufu, n);
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 2;
}
