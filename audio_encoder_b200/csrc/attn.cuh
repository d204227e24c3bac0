// Windowed (block-diagonal) self-attention (page "MOSS-Transcribe-preview-2B -
// GGUF", "Architecture" table, Audio encoder row): every token attends only
// the tokens of its own window (one 800-frame chunk, at most 100 tokens).
//
// One CTA per (window, head).  The window's Q, K, V slices (<= 128 rows x 64)
// are staged in shared memory; each of 8 warps owns 16 query rows, computes
// S = Q K^T / 8 with bf16 tensor-core MMAs, an fp32 softmax in registers
// (keys past the window length masked), and O = P V.  Nothing crosses
// windows, so windows never exchange data.
#pragma once

#include "common.cuh"

namespace moss {

static constexpr int ATTN_MAX_WIN = 128;
static constexpr int ATTN_PITCH = 72;  // bf16 per shared row (144 B: conflict-free ldmatrix)
static constexpr size_t ATTN_SMEM = 3 * ATTN_MAX_WIN * ATTN_PITCH * sizeof(bf16);

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// qkv [T][3840] bf16 = q | k | v (each 20 heads x 64); out [T][1280] bf16.
// windows[w] = {first token, tokens} with 1 <= tokens <= 128.
__global__ void __launch_bounds__(256) window_attn_kernel(const bf16 *__restrict__ qkv,
                                                          const int2 *__restrict__ windows,
                                                          bf16 *__restrict__ out)
{
    extern __shared__ __align__(16) uint8_t attn_smem[];
    bf16 *Qs = reinterpret_cast<bf16 *>(attn_smem);
    bf16 *Ks = Qs + ATTN_MAX_WIN * ATTN_PITCH;
    bf16 *Vs = Ks + ATTN_MAX_WIN * ATTN_PITCH;
    const int h = blockIdx.y;
    const int2 win = windows[blockIdx.x];
    const int s = win.x, n = win.y;
    const int tid = threadIdx.x;

    for (int i = tid; i < 3 * ATTN_MAX_WIN * 8; i += 256) {
        const int mat = i / (ATTN_MAX_WIN * 8), r = (i / 8) % ATTN_MAX_WIN, c8 = i % 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < n) v = *reinterpret_cast<const uint4 *>(qkv + (size_t)(s + r) * 3840 + mat * 1280 + h * 64 + c8 * 8);
        *reinterpret_cast<uint4 *>(Qs + (size_t)mat * ATTN_MAX_WIN * ATTN_PITCH + r * ATTN_PITCH + c8 * 8) = v;
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    const int r0 = warp * 16;
    if (r0 >= n) return;
    const int nkb = (n + 15) >> 4;  // key blocks of 16

    uint32_t qf[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; kk++)
        ldsm_x4(qf[kk], Qs + (r0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ATTN_PITCH + kk * 16 + 8 * (lane >> 4));

    float sc[16][4];
#pragma unroll
    for (int j = 0; j < 16; j++) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.0f;
#pragma unroll
    for (int jb = 0; jb < 8; jb++) {
        if (jb < nkb) {
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
                uint32_t b[4];
                ldsm_x4(b, Ks + (jb * 16 + (lane & 7) + 8 * (lane >> 4)) * ATTN_PITCH + kk * 16 + 8 * ((lane >> 3) & 1));
                mma16816(sc[2 * jb], qf[kk], b[0], b[1]);
                mma16816(sc[2 * jb + 1], qf[kk], b[2], b[3]);
            }
        }
    }

    const float scale = 0.125f * 1.4426950408889634f;  // 1/sqrt(64) in base-2 exponent units
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; j++) {
        if (j < 2 * nkb) {
            const int key = 8 * j + 2 * (lane & 3);
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const bool ok = key + e < n;
                sc[j][e] = ok ? sc[j][e] * scale : -INFINITY;
                sc[j][2 + e] = ok ? sc[j][2 + e] * scale : -INFINITY;
            }
            mx0 = fmaxf(mx0, fmaxf(sc[j][0], sc[j][1]));
            mx1 = fmaxf(mx1, fmaxf(sc[j][2], sc[j][3]));
        }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    float sum0 = 0.0f, sum1 = 0.0f;
    uint32_t pa[8][4];
#pragma unroll
    for (int j = 0; j < 16; j++) {
        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
        if (j < 2 * nkb) {
            p0 = exp2f(sc[j][0] - mx0);
            p1 = exp2f(sc[j][1] - mx0);
            p2 = exp2f(sc[j][2] - mx1);
            p3 = exp2f(sc[j][3] - mx1);
        }
        sum0 += p0 + p1;
        sum1 += p2 + p3;
        pa[j >> 1][(j & 1) * 2] = pack_bf16x2(p0, p1);
        pa[j >> 1][(j & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        sum0 += __shfl_xor_sync(0xffffffffu, sum0, o);
        sum1 += __shfl_xor_sync(0xffffffffu, sum1, o);
    }

    float oacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; j++) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.0f;
#pragma unroll
    for (int kb = 0; kb < 8; kb++) {
        if (kb < nkb) {
#pragma unroll
            for (int dp = 0; dp < 4; dp++) {
                uint32_t b[4];
                ldsm_x4_t(b, Vs + (kb * 16 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ATTN_PITCH + dp * 16 + 8 * (lane >> 4));
                mma16816(oacc[2 * dp], pa[kb], b[0], b[1]);
                mma16816(oacc[2 * dp + 1], pa[kb], b[2], b[3]);
            }
        }
    }

    const float inv0 = 1.0f / sum0, inv1 = 1.0f / sum1;
    const int ra = r0 + (lane >> 2), rb = ra + 8;
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const int d = h * 64 + 8 * j + 2 * (lane & 3);
        if (ra < n)
            *reinterpret_cast<uint32_t *>(out + (size_t)(s + ra) * 1280 + d) = pack_bf16x2(oacc[j][0] * inv0, oacc[j][1] * inv0);
        if (rb < n)
            *reinterpret_cast<uint32_t *>(out + (size_t)(s + rb) * 1280 + d) = pack_bf16x2(oacc[j][2] * inv1, oacc[j][3] * inv1);
    }
}

}  // namespace moss
