// Conv2D stem helpers (page "MOSS-Transcribe-preview-2B - GGUF",
// "Architecture" table, Conv front-end row): conv1 (1 -> 480 channels, 3x3,
// stride 2, padding 1, GELU) as a K = 32 GEMM on the tensor cores.  conv2 and
// conv3 are implicit GEMMs on the tensor cores (gemm.cuh, A_CONV_S2).
//
// Activations are NHWC per 800-frame chunk: [chunk][time][freq][480] bf16.
#pragma once

#include "common.cuh"

namespace moss {

struct StemChunk {
    int clip;       // clip slot (for the log-mel maximum)
    int mel_row;    // first row of this chunk in the raw log-mel buffer
    int nframes;    // valid frames (1..800); the rest of the chunk is zero
    int t1_lim;     // conv1 output time steps the chunk's tokens need (<= 400)
};

// conv1 over the normalised log-mel of a chunk as a small GEMM on the tensor
// cores.  Input plane (freq 128, time 800), with frames >= nframes zero (the
// tail padding) and conv padding 1.  Output [chunk][400][64][480] bf16, GELU
// applied.
//
// A tile is 128 output pixels (time steps t0, t0 + 1 x all 64 frequencies;
// row m = 64 (t - t0) + f) by all 480 channels, computed as two N = 240
// halves into two TMEM accumulators (columns 0 and 256).  The GEMM's K row of
// a pixel holds its nine input taps split into bf16 pairs, then a 1.0:
//   k 0..8 = hi(x_tap), k 9..17 = lo(x_tap) = bf16(x - hi), k 18 = 1, rest 0
// (tap = 3 kf + kt), against the weight row [w_tap, w_tap, bias, 0...] of each
// channel (the weights and bias are bf16 numbers, so the products are exact
// and the split keeps x to ~2^-16), K = 32 in two MMA k-steps.  Persistent
// CTAs walk the (chunk, tile) items:
//   warps 0-3 (builders): the tile's five input frames into shared memory,
//     normalised on load; thread m then writes K row m of the A tile
//     (128-byte swizzled rows, double-buffered); thread 0 issues the MMAs;
//   warps 4-15 (epilogue): three warps per TMEM lane quarter, 80 channels
//     each: GELU on the accumulators, bf16 into the warp's staging area
//     (32 pixels x 160 bytes), out by one TMA store (a pixel's channels are
//     960 bytes apart from the next pixel's, so per-lane stores would each
//     touch their own line).
// The weights (B, [480][64] bf16, swizzled on the host) stay in shared
// memory for the CTA's life.
static constexpr int C1_BUILD_WARPS = 4, C1_EPI_WARPS = 12;
static constexpr int C1_THREADS = 32 * (C1_BUILD_WARPS + C1_EPI_WARPS);
static constexpr uint32_t C1_B_BYTES = 480 * 128;  // weights, K-major, 128-byte swizzle
static constexpr uint32_t C1_A_BYTES = 128 * 128;  // one A tile
static constexpr uint32_t C1_PLANE_OFF = C1_B_BYTES + 2 * C1_A_BYTES;
static constexpr uint32_t C1_STG_OFF = (C1_PLANE_OFF + 5 * 132 * 4 + 1023) / 1024 * 1024;
static constexpr uint32_t C1_STG_BYTES = 32 * 80 * 2;  // one epilogue warp's box
static constexpr uint32_t C1_BAR_OFF = C1_STG_OFF + C1_EPI_WARPS * C1_STG_BYTES;
static constexpr size_t C1_SMEM = 1024 + C1_BAR_OFF + 64;
static_assert(C1_B_BYTES % 1024 == 0 && (240 * 128) % 1024 == 0, "operand tiles keep the swizzle alignment");

__global__ void __launch_bounds__(C1_THREADS, 1) conv1_tc_kernel(const float *__restrict__ mel_raw,
                                                                 const StemChunk *__restrict__ chunks, int n_chunks,
                                                                 const int *__restrict__ gmax_ord,
                                                                 const uint4 *__restrict__ wB,  // [480][64] swizzled
                                                                 const __grid_constant__ CUtensorMap tm_out,
                                                                 int *err)
{
    extern __shared__ uint8_t c1_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(c1_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sB = sm, *sA = sm + C1_B_BYTES;
    float(*plane)[132] = reinterpret_cast<float(*)[132]>(sm + C1_PLANE_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C1_BAR_OFF);
    uint64_t *a_empty = bars, *t_full = bars + 2, *t_empty = bars + 4;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 6);
    volatile int *build_ok = reinterpret_cast<volatile int *>(bars + 7);  // builders: cleared when a wait gives up
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) prefetch_tmap(&tm_out);

    // the weights do not depend on earlier kernels
    for (int i = tid; i < (int)(C1_B_BYTES / 16); i += C1_THREADS) reinterpret_cast<uint4 *>(sB)[i] = wB[i];
    fence_async_smem();  // generic stores, read by the MMA
    if (tid == 0) {
        for (int i = 0; i < 2; i++) {
            mbar_init(&a_empty[i], 1);
            mbar_init(&t_full[i], 1);
            mbar_init(&t_empty[i], C1_EPI_WARPS);
        }
        fence_mbar_init();
        *build_ok = 1;
    }
    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    grid_dep_launch();  // this CTA holds its TMEM
    grid_dep_wait();    // the log-mel rows and the clip maxima are written

    const int n_items = n_chunks * 200;
    bool ok = true;
    int last_b = -1;  // thread 0: buffer and phase parity of its last commit
    uint32_t last_par = 0;
    if (warp < C1_BUILD_WARPS) {
        // The builders pass two named barriers per tile and must all leave the
        // loop at the same tile: a failed wait clears build_ok, which every
        // builder reads right after the next barrier.
        const int m = tid, tl = m >> 6, f = m & 63;
        constexpr uint32_t idesc = idesc_bf16(128, 240);
        int i = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
            const int ci = item / 200, t0 = 2 * (item - 200 * ci);
            const StemChunk ch = chunks[ci];
            if (t0 >= ch.t1_lim) continue;  // outside the receptive field of the chunk's tokens
            const int b = i & 1;
            uint8_t *A = sA + b * C1_A_BYTES;
            if (!mbar_wait(&a_empty[b], ((i >> 1) & 1) ^ 1, err)) *build_ok = 0;
            // the five input frames 2 t0 - 1 .. 2 t0 + 3, column 2 + f = frequency f
            const float floor_v = ordered_to_float(gmax_ord[ch.clip]) - 8.0f;
            for (int j = m; j < 5 * 132; j += 32 * C1_BUILD_WARPS) {
                const int r = j / 132, col = j - 132 * r, fi = col - 2;
                const int ti = 2 * t0 - 1 + r;
                float v = 0.0f;
                if (fi >= 0 && fi < 128 && ti >= 0 && ti < ch.nframes) {
                    const float x = mel_raw[(size_t)(ch.mel_row + ti) * 128 + fi];
                    v = (fmaxf(x, floor_v) + 4.0f) * 0.25f;
                }
                plane[r][col] = v;
            }
            named_bar_sync(1, 32 * C1_BUILD_WARPS);
            if (!*build_ok) break;
            // K row m: taps (kf, kt) = frequency 2 f - 1 + kf, frame 2 t - 1 + kt
            uint32_t hv[9];
            float lv[9];
#pragma unroll
            for (int kf = 0; kf < 3; kf++)
#pragma unroll
                for (int kt = 0; kt < 3; kt++) {
                    const float x = plane[2 * tl + kt][2 * f + 1 + kf];
                    const bf16 hi = __float2bfloat16_rn(x);
                    hv[3 * kf + kt] = (uint32_t)__bfloat16_as_ushort(hi);
                    lv[3 * kf + kt] = x - __bfloat162float(hi);
                }
            uint32_t w[16];
            auto lo16 = [&](int t) { return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lv[t])); };
            w[0] = hv[0] | hv[1] << 16;
            w[1] = hv[2] | hv[3] << 16;
            w[2] = hv[4] | hv[5] << 16;
            w[3] = hv[6] | hv[7] << 16;
            w[4] = hv[8] | lo16(0) << 16;
            w[5] = lo16(1) | lo16(2) << 16;
            w[6] = lo16(3) | lo16(4) << 16;
            w[7] = lo16(5) | lo16(6) << 16;
            w[8] = lo16(7) | lo16(8) << 16;
            w[9] = 0x3F80u;  // k 18 = 1.0 (bias), k 19 = 0
#pragma unroll
            for (int q = 10; q < 16; q++) w[q] = 0;
            uint8_t *row = A + m * 128;
#pragma unroll
            for (int c = 0; c < 4; c++)
                *reinterpret_cast<uint4 *>(row + ((c ^ (m & 7)) << 4)) = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            fence_async_smem();
            named_bar_sync(1, 32 * C1_BUILD_WARPS);
            if (tid == 0) {
                for (int h = 0; h < 2; h++) {
                    if (!mbar_wait(&t_empty[h], (i & 1) ^ 1, err)) {
                        *build_ok = 0;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(smem_u32(A)), bd = sw128_desc(smem_u32(sB + h * 240 * 128));
                    mma_bf16(tbase + 256 * h, ad, bd, idesc, 0);
                    mma_bf16(tbase + 256 * h, ad + 2, bd + 2, idesc, 1);  // k 16..31: +32 bytes
                    mma_commit(&t_full[h]);
                }
                mma_commit(&a_empty[b]);  // the A tile is read once both halves are done
                last_b = b;
                last_par = (i >> 1) & 1;
            }
            i++;
        }
    } else {
        // output map: [chunk * 400 * 64 + t * 64 + f][480] bf16, boxes of 80
        // channels x 32 pixels, no swizzle
        const int e = warp - C1_BUILD_WARPS, q = warp & 3, g = e >> 2;
        const int tl = q >> 1;  // the warp's 32 pixels: time step t0 + tl, frequencies 32 (q & 1) ..
        uint8_t *stg = sm + C1_STG_OFF + e * C1_STG_BYTES + lane * 160;
        int i = 0;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const int ci = item / 200, t0 = 2 * (item - 200 * ci);
            const StemChunk ch = chunks[ci];
            if (t0 >= ch.t1_lim) continue;
            const bool live = t0 + tl < ch.t1_lim;  // the whole warp's time step
            for (int h = 0; h < 2; h++) {
                if (!mbar_wait(&t_full[h], i & 1, err)) { ok = false; break; }
                tc_fence_after();
                if (live) {
                    if (lane == 0) bulk_wait_read();  // the previous box has left the staging area
                    __syncwarp();
                    const uint32_t ta = tbase + ((uint32_t)(q * 32) << 16) + 256 * h + 80 * g;
#pragma unroll
                    for (int piece = 0; piece < 3; piece++) {
                        uint32_t r[32];
                        if (piece < 2)
                            tmem_ld32(ta + 32 * piece, r);
                        else
                            tmem_ld16(ta + 64, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 4; c++) {
                            if (piece == 2 && c >= 2) break;
                            uint32_t pk[4];
#pragma unroll
                            for (int j = 0; j < 4; j++) {
                                const float2 y = gelu2(make_float2(__uint_as_float(r[8 * c + 2 * j]),
                                                                   __uint_as_float(r[8 * c + 2 * j + 1])));
                                pk[j] = pack_bf16x2(y.x, y.y);
                            }
                            *reinterpret_cast<uint4 *>(stg + 64 * piece + 16 * c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&t_empty[h]);  // the accumulator is read
                if (live) {
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int row0 = (ci * 400 + t0 + tl) * 64 + 32 * (q & 1);
                        tma_store_2d(&tm_out, sm + C1_STG_OFF + e * C1_STG_BYTES, 240 * h + 80 * g, row0);
                        bulk_commit();
                    }
                }
            }
            i++;
        }
        if (lane == 0) bulk_wait_all();  // the warp's boxes are written before the grid ends
    }
    // a wait that gave up can leave MMAs in flight: let them land (bounded)
    // before the TMEM columns are released
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *(volatile int *)err != 0 && last_b >= 0) mbar_drain(&a_empty[last_b], last_par);
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace moss
