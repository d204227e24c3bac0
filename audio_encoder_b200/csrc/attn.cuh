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
// is TMEM lane i.  TMA brings the 128-row Q, K and V slices of the window
// (rows past the window belong to the next window or lie past the end and are
// masked / zero).  S = Q K^T (M = N = 128, K = 64) accumulates in TMEM; each
// thread reads its row of S, masks keys past the window, and writes
// P = exp(S/8 - max) as bf16 into shared memory in the swizzled K-major layout
// (over the Q and K slots, which are free once S is done).  O = P V (M = 128,
// N = 64, K = 128) takes V straight from its TMA layout as an MN-major
// operand, lands in TMEM, and is scaled by 1 / rowsum on the way out.
static constexpr size_t ATTN_TC_SMEM = 1024 + 3 * 16384 + 64;

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

__global__ void __launch_bounds__(128) window_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                                                             const int2 *__restrict__ windows,
                                                             bf16 *__restrict__ out, int *err)
{
    extern __shared__ uint8_t attn_tc_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(attn_tc_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = sm, *sK = sm + 16384, *sV = sm + 32768;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 49152);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);
    const int h = blockIdx.y;
    const int2 win = windows[blockIdx.x];  // host-written table
    const int s = win.x, n = win.y;
    const int tid = threadIdx.x, warp = tid >> 5;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        prefetch_tmap(&tm_qkv);
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
    // the TMEM of this CTA is held: later kernels may start (they never wait
    // for TMEM that an unstarted CTA of this grid would need)
    grid_dep_launch();
    grid_dep_wait();

    if (tid == 0) {
        mbar_arrive_expect_tx(&bars[0], 3 * 16384);
        tma_load_2d(&tm_qkv, &bars[0], sQ, h * 64, s);
        tma_load_2d(&tm_qkv, &bars[0], sK, 1280 + h * 64, s);
        tma_load_2d(&tm_qkv, &bars[0], sV, 2560 + h * 64, s);
        if (mbar_wait(&bars[0], 0, err)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16(128, 128);
#pragma unroll
            for (int k = 0; k < 4; k++)
                mma_bf16(tbase, sw128_desc(smem_u32(sQ) + 32 * k), sw128_desc(smem_u32(sK) + 32 * k), idesc, k > 0);
            mma_commit(&bars[1]);
        }
    }
    bool ok = mbar_wait(&bars[1], 0, err);
    tc_fence_after();

    // softmax of this thread's row (keys >= n masked); P to shared memory
    const float scale = 0.125f * 1.4426950408889634f;
    float mx = -INFINITY;
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; j++)
            if (c0 + j < n) mx = fmaxf(mx, __uint_as_float(v[j]) * scale);
    }
    float sum = 0.0f;
    const int r = tid, sw = r & 7;
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(trow + c0, v);
        tmem_ld_wait();
        uint8_t *blk = (c0 < 64 ? sQ : sK) + r * 128;
#pragma unroll
        for (int q = 0; q < 4; q++) {
            float p[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int key = c0 + 8 * q + j;
                p[j] = key < n ? exp2f(__uint_as_float(v[8 * q + j]) * scale - mx) : 0.0f;
                sum += p[j];
            }
            const int chunk16 = ((c0 & 63) >> 3) + q;  // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4 *>(blk + ((chunk16 ^ sw) << 4)) =
                make_uint4(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]),
                           pack_bf16x2(p[6], p[7]));
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (tid == 0 && ok) {
        constexpr uint32_t idesc = idesc_bf16(128, 64) | (1u << 16);  // B (V) is MN-major
#pragma unroll
        for (int ks = 0; ks < 8; ks++) {
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
        uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)(s + r) * 1280 + h * 64);
#pragma unroll
        for (int q = 0; q < 4; q++)
            dst[q] = make_uint4(pack_bf16x2(__uint_as_float(o0[8 * q]) * inv, __uint_as_float(o0[8 * q + 1]) * inv),
                                pack_bf16x2(__uint_as_float(o0[8 * q + 2]) * inv, __uint_as_float(o0[8 * q + 3]) * inv),
                                pack_bf16x2(__uint_as_float(o0[8 * q + 4]) * inv, __uint_as_float(o0[8 * q + 5]) * inv),
                                pack_bf16x2(__uint_as_float(o0[8 * q + 6]) * inv, __uint_as_float(o0[8 * q + 7]) * inv));
#pragma unroll
        for (int q = 0; q < 4; q++)
            dst[4 + q] = make_uint4(pack_bf16x2(__uint_as_float(o1[8 * q]) * inv, __uint_as_float(o1[8 * q + 1]) * inv),
                                    pack_bf16x2(__uint_as_float(o1[8 * q + 2]) * inv, __uint_as_float(o1[8 * q + 3]) * inv),
                                    pack_bf16x2(__uint_as_float(o1[8 * q + 4]) * inv, __uint_as_float(o1[8 * q + 5]) * inv),
                                    pack_bf16x2(__uint_as_float(o1[8 * q + 6]) * inv, __uint_as_float(o1[8 * q + 7]) * inv));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 128);
}

}  // namespace moss
