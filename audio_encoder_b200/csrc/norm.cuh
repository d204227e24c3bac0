// LayerNorm over rows of 1280 fp32 (the residual stream) into bf16 GEMM
// operands: y = (x - mean) / sqrt(var + 1e-5) * gamma + beta, statistics in
// fp32 with the variance taken around the mean (two passes over registers).
// One warp per row; each lane holds 40 values as 10 float4.
#pragma once

#include "common.cuh"

namespace moss {

__global__ void __launch_bounds__(256) layernorm1280_kernel(const float *__restrict__ x,
                                                            const float *__restrict__ gamma,
                                                            const float *__restrict__ beta,
                                                            bf16 *__restrict__ y, int rows)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= rows) return;
    const float4 *xr = reinterpret_cast<const float4 *>(x + (size_t)warp * 1280);
    float4 v[10];
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 10; i++) {
        v[i] = xr[lane + 32 * i];
        s += v[i].x + v[i].y + v[i].z + v[i].w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s * (1.0f / 1280.0f);
    float q = 0.0f;
#pragma unroll
    for (int i = 0; i < 10; i++) {
        const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
        q += a * a + b * b + c * c + d * d;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = rsqrtf(q * (1.0f / 1280.0f) + 1e-5f);
    const float4 *g4 = reinterpret_cast<const float4 *>(gamma);
    const float4 *b4 = reinterpret_cast<const float4 *>(beta);
    uint2 *yr = reinterpret_cast<uint2 *>(y + (size_t)warp * 1280);
#pragma unroll
    for (int i = 0; i < 10; i++) {
        const float4 g = g4[lane + 32 * i], b = b4[lane + 32 * i];
        uint2 o;
        o.x = pack_bf16x2((v[i].x - mean) * rstd * g.x + b.x, (v[i].y - mean) * rstd * g.y + b.y);
        o.y = pack_bf16x2((v[i].z - mean) * rstd * g.z + b.z, (v[i].w - mean) * rstd * g.w + b.w);
        yr[lane + 32 * i] = o;
    }
}

}  // namespace moss
