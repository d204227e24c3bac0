// LayerNorm over rows of 1280 fp32 (the residual stream) into bf16 GEMM
// operands: y = (x - mean) / sqrt(var + 1e-5) * gamma + beta, statistics in
// fp32 with the variance taken around the mean (two passes over registers).
// One warp per row; each lane holds 40 values as 10 float4.  With split set,
// row r is written as hi = bf16(y) at [r][c] and lo = bf16(y - hi) at
// [r][1280 + c] (row stride ldy), for GEMMs that take [hi | lo].
#pragma once

#include "common.cuh"

namespace moss {

__global__ void __launch_bounds__(256, 4) layernorm1280_kernel(const float *__restrict__ x,
                                                            const float *__restrict__ gamma,
                                                            const float *__restrict__ beta,
                                                            bf16 *__restrict__ y, int rows, int ldy,
                                                            int split)
{
    grid_dep_wait();
    grid_dep_launch();
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
    uint2 *yr = reinterpret_cast<uint2 *>(y + (size_t)warp * ldy);
    uint2 *yl = reinterpret_cast<uint2 *>(y + (size_t)warp * ldy + 1280);
#pragma unroll
    for (int i = 0; i < 10; i++) {
        const float4 g = g4[lane + 32 * i], b = b4[lane + 32 * i];
        const float a0 = (v[i].x - mean) * rstd * g.x + b.x, a1 = (v[i].y - mean) * rstd * g.y + b.y;
        const float a2 = (v[i].z - mean) * rstd * g.z + b.z, a3 = (v[i].w - mean) * rstd * g.w + b.w;
        uint2 o;
        o.x = pack_bf16x2(a0, a1);
        o.y = pack_bf16x2(a2, a3);
        yr[lane + 32 * i] = o;
        if (split) {
            const __nv_bfloat162 h01 = *reinterpret_cast<const __nv_bfloat162 *>(&o.x);
            const __nv_bfloat162 h23 = *reinterpret_cast<const __nv_bfloat162 *>(&o.y);
            uint2 l;
            l.x = pack_bf16x2(a0 - __low2float(h01), a1 - __high2float(h01));
            l.y = pack_bf16x2(a2 - __low2float(h23), a3 - __high2float(h23));
            yl[lane + 32 * i] = l;
        }
    }
}

}  // namespace moss
