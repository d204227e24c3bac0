// Windowed (block-diagonal) self-attention (page "MOSS-Transcribe-preview-2B -
// GGUF", "Architecture" table, Audio encoder row): every token attends only
// the tokens of its own window (one 800-frame chunk, at most 100 tokens).
//
// Windows hold at most 128 tokens (here 100); nothing crosses windows, so
// windows never exchange data.
#pragma once

#include "common.cuh"

namespace moss {

// One CTA of 128 threads per (window, head); thread i owns query row i, which
// is TMEM lane i.  Windows hold at most ATTN_ROWS = 112 tokens (here 100).
// TMA brings 112-row Q, K and V slices of the window (rows past the window
// belong to the next window or lie past the end, read as zeros); each slice
// is 14 KB, so five CTAs fit on an SM.  S = Q K^T (M = 128, N = 112, K = 64)
// accumulates in TMEM; the MMA's query rows 112..127 read the start of the K
// slice and give rows that are never used.  Each thread reads its row of S,
// masks keys past the window, and writes P = 2^(S log2(e)/8 - max) as bf16 in
// the swizzled K-major layout over the Q slot (keys 0..63) and the K slot
// (keys 64..111), both free once S is done.  O = P V (M = 128, N = 64,
// K = 112) takes V straight from its TMA layout as an MN-major operand, lands
// in TMEM, and is scaled by 1 / rowsum on the way out.
static constexpr int ATTN_ROWS = 112;
static constexpr uint32_t ATTN_SLICE = ATTN_ROWS * 128;  // bytes of one 112 x 64 bf16 slice
static constexpr size_t ATTN_TC_SMEM = 1024 + 3 * ATTN_SLICE + 64;

// Shared-memory descriptor of an MN-major operand with 128-byte swizzle:
// rows of 64 bf16 along N (128 B) for consecutive K, 8-row K groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t smem_addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(1024 >> 4) << 32;  // stride between 8-row groups along K
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// 2^x by the special-function unit (PTX ex2.approx: relative error about
// 2^-22, far below the bf16 rounding of the probabilities it feeds).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// p = 2^(s * scale + off) for NV consecutive scores of this thread's row
// (keys c0 ..), zero for keys >= n, summed into sum2 and written as bf16 to
// the 16-byte chunks 0 .. NV/8-1 of the row's 128-byte K-major line.
template <int NV>
__device__ __forceinline__ void softmax_part(const uint32_t *v, int c0, int n, float2 sc2, float2 off2, float2 &sum2,
                                             uint8_t *line, int sw)
{
    const bool full = c0 + NV <= n;
#pragma unroll
    for (int q = 0; q < NV / 8; q++) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int k0 = 8 * q + 2 * j;
            const float2 t = __ffma2_rn(make_float2(__uint_as_float(v[k0]), __uint_as_float(v[k0 + 1])), sc2, off2);
            float2 e = make_float2(ex2_approx(t.x), ex2_approx(t.y));
            if (!full) {
                if (c0 + k0 >= n) e.x = 0.0f;
                if (c0 + k0 + 1 >= n) e.y = 0.0f;
            }
            sum2 = __fadd2_rn(sum2, e);
            w[j] = pack_bf16x2(e.x, e.y);
        }
        *reinterpret_cast<uint4 *>(line + ((q ^ sw) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__global__ void __launch_bounds__(128) window_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                                                             const int2 *__restrict__ windows,
                                                             bf16 *__restrict__ out, int *err)
{
    extern __shared__ uint8_t attn_tc_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(attn_tc_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = sm, *sK = sm + ATTN_SLICE, *sV = sm + 2 * ATTN_SLICE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 3 * ATTN_SLICE);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);
    const int h = blockIdx.y;
    const int2 win = windows[blockIdx.x];  // host-written table
    const int s = win.x, n = win.y;
    const int tid = threadIdx.x, warp = tid >> 5;

    // The loads go out before the TMEM allocation, which may wait for other
    // CTAs on this SM to free theirs (TMEM holds four of these CTAs' 128
    // columns; shared memory holds five).
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        prefetch_tmap(&tm_qkv);
        grid_dep_wait();
        mbar_arrive_expect_tx(&bars[0], 3 * ATTN_SLICE);
        tma_load_2d(&tm_qkv, &bars[0], sQ, h * 64, s);
        tma_load_2d(&tm_qkv, &bars[0], sK, 1280 + h * 64, s);
        tma_load_2d(&tm_qkv, &bars[0], sV, 2560 + h * 64, s);
    }
    if (warp == 0) {
        tmem_alloc(tslot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t trow = tbase + ((uint32_t)(warp * 32) << 16);
    // this CTA holds its TMEM: later kernels may start (none of them then
    // holds TMEM that a CTA of this grid still waits for)
    grid_dep_launch();
    grid_dep_wait();

    if (tid == 0) {
        if (mbar_wait(&bars[0], 0, err)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16(128, ATTN_ROWS);
#pragma unroll
            for (int k = 0; k < 4; k++)
                mma_bf16(tbase, sw128_desc(smem_u32(sQ) + 32 * k), sw128_desc(smem_u32(sK) + 32 * k), idesc, k > 0);
            mma_commit(&bars[1]);
        }
    }
    bool ok = mbar_wait(&bars[1], 0, err);
    tc_fence_after();

    // softmax of this thread's row.  Pass 1: the row maximum of the raw scores
    // (the scale is positive); pass 2: p in pairs, summed, written as bf16.
    // A part of the row wholly past the window is skipped (its P chunks are
    // zeros that no MMA step reads past key n: see below).
    const float scale = 0.125f * 1.4426950408889634f;
    const int r = tid, sw = r & 7;
    float mx = -INFINITY;
    {
        uint32_t v[64];
        tmem_ld32(trow, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(trow + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        if (n >= 64) {
#pragma unroll
            for (int j = 0; j < 64; j++) mx = fmaxf(mx, __uint_as_float(v[j]));
        } else {
#pragma unroll
            for (int j = 0; j < 64; j++)
                if (j < n) mx = fmaxf(mx, __uint_as_float(v[j]));
        }
        if (n > 64) {
            tmem_ld32(trow + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld16(trow + 96, &v[32]);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 48; j++)
                if (64 + j < n) mx = fmaxf(mx, __uint_as_float(v[j]));
        }
    }
    const float2 sc2 = make_float2(scale, scale), off2 = make_float2(-mx * scale, -mx * scale);
    float2 sum2 = make_float2(0.0f, 0.0f);
    {
        uint32_t v[64];
        tmem_ld32(trow, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(trow + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        const bool own = r < ATTN_ROWS;  // rows 112..127 of P overlap the next slot: never written
        if (own) softmax_part<64>(v, 0, n, sc2, off2, sum2, sQ + r * 128, sw);
        if (n > 64) {
            tmem_ld32(trow + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld16(trow + 96, &v[32]);
            tmem_ld_wait();
            if (own) softmax_part<48>(v, 64, n, sc2, off2, sum2, sK + r * 128, sw);
        }
    }
    const float sum = sum2.x + sum2.y;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // O = P V over the key steps that hold keys < n (P holds zeros between n
    // and the end of its last step; V rows there are finite)
    if (tid == 0 && ok) {
        constexpr uint32_t idesc = idesc_bf16(128, 64) | (1u << 16);  // B (V) is MN-major
        const int ksteps = (n + 15) >> 4;                             // <= 7
        for (int ks = 0; ks < ksteps; ks++) {
            const uint32_t a = smem_u32(ks < 4 ? sQ : sK) + 32 * (ks & 3);
            mma_bf16(tbase, sw128_desc(a), sw128_mn_desc(smem_u32(sV) + 2048 * ks), idesc, ks > 0);
        }
        mma_commit(&bars[1]);
    }
    ok = mbar_wait(&bars[1], 1, err) && ok;
    tc_fence_after();
    uint32_t o0[32], o1[32];
    tmem_ld32(trow, o0);
    tmem_ld32(trow + 32, o1);
    tmem_ld_wait();
    if (ok && r < n) {
        const float inv = 1.0f / sum;
        const float2 inv2 = make_float2(inv, inv);
        uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)(s + r) * 1280 + h * 64);
#pragma unroll
        for (int q = 0; q < 8; q++) {
            const uint32_t *o = q < 4 ? &o0[8 * q] : &o1[8 * (q - 4)];
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const float2 y = __fmul2_rn(make_float2(__uint_as_float(o[2 * j]), __uint_as_float(o[2 * j + 1])), inv2);
                w[j] = pack_bf16x2(y.x, y.y);
            }
            dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 128);
}

}  // namespace moss
