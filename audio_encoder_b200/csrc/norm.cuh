// LayerNorm over rows of 1280 fp32 (the residual stream) into bf16 GEMM
// operands: y = (x - mean) / sqrt(var + 1e-5) * gamma + beta, statistics in
// fp32 with the variance taken around the mean (two passes over registers).
// One warp per row; each lane holds 40 values as 10 float4.  With split set,
// row r is written as hi = bf16(y) at [r][c] and lo = bf16(y - hi) at
// [r][1280 + c] (row stride ldy), for GEMMs that take [hi | lo].
#pragma once

#include <cuda_fp8.h>

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

// The same LayerNorm into e4m3 GEMM operands: the row's values y as above,
// then s = max |y| / 448 (fp32) and y8 = e4m3(y / s) (fp32 division, round to
// nearest even, saturating), s to row_scale[r] (0 and zero operands for a
// zero row).  The GEMM multiplies its row by s again.
__global__ void __launch_bounds__(256, 3) layernorm1280_e4m3_kernel(const float *__restrict__ x,
                                                                 const float *__restrict__ gamma,
                                                                 const float *__restrict__ beta,
                                                                 uint8_t *__restrict__ y8, float *__restrict__ row_scale,
                                                                 int rows)
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
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 10; i++) {
        const float4 g = g4[lane + 32 * i], b = b4[lane + 32 * i];
        v[i].x = (v[i].x - mean) * rstd * g.x + b.x;
        v[i].y = (v[i].y - mean) * rstd * g.y + b.y;
        v[i].z = (v[i].z - mean) * rstd * g.z + b.z;
        v[i].w = (v[i].w - mean) * rstd * g.w + b.w;
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = amax / 448.0f;
    if (lane == 0) row_scale[warp] = sc;
    uint32_t *yr = reinterpret_cast<uint32_t *>(y8 + (size_t)warp * 1280);
#pragma unroll
    for (int i = 0; i < 10; i++) {
        uint32_t packed = 0;
        if (sc > 0.0f) {
            const __nv_fp8x2_storage_t p01 =
                __nv_cvt_float2_to_fp8x2(make_float2(v[i].x / sc, v[i].y / sc), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t p23 =
                __nv_cvt_float2_to_fp8x2(make_float2(v[i].z / sc, v[i].w / sc), __NV_SATFINITE, __NV_E4M3);
            packed = (uint32_t)p01 | ((uint32_t)p23 << 16);
        }
        yr[lane + 32 * i] = packed;
    }
}

}  // namespace moss
