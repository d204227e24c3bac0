// Persistent, warp-specialised bf16 GEMM on the 5th-generation tensor cores.
//
//   C[M][N] = A[M][K] * B[N][K]^T   (A, B K-major bf16; fp32 accumulate in TMEM)
//
// One CTA per SM walks output tiles of 128 x BN.  Warp 0 (one lane) streams
// 128x64 A and BNx64 B tiles with TMA into a ring of shared-memory stages;
// warp 1 (one lane) issues tcgen05.mma (M=128, N=BN, K=16) into one of two
// TMEM accumulators; warps 2-9 drain the other accumulator with tcgen05.ld
// and apply the fused epilogue (bias, GELU, residual add, SwiGLU, conv_out
// row packing + positions) while the next tile's mainloop runs.  A warp may
// only read the TMEM lane quarter (warp id mod 4), so two epilogue warps share
// each quarter and split the tile's 32-column chunks between them.
#pragma once

#include "common.cuh"

namespace moss {

enum EpiKind : int {
    EPI_BF16 = 0,       // out bf16 = acc + bias
    EPI_GELU_BF16 = 1,  // out bf16 = GELU(acc + bias)
    EPI_RESID_F32 = 2,  // out fp32 += acc + bias          (residual stream)
    EPI_SWIGLU_BF16 = 3,// columns interleaved in 32s: gate, up -> out = SiLU(g) * u
    EPI_CONVOUT_F32 = 4,// row r of chunk r/100: out[tok0 + r%100] = acc + pos[r%100]
    EPI_F32 = 5         // out fp32 = acc + bias
};

// How the A operand is fetched.
enum AMode : int {
    A_PLAIN = 0,    // A [M][K] row-major, 2-D tensor map
    A_CONV_S2 = 1   // implicit 3x3 / stride 2 / pad 1 conv over NHWC [chunk][T][F][480]:
                    // k-block kb = tap*8 + channel block, tap = kf*3 + kt
};

struct GemmArgs {
    int M, N, K;
    int m_tiles, n_tiles;
    int *err;
    const float *bias;      // [N] (EPI_CONVOUT: unused)
    void *out;              // output base
    int ldo;                // output leading dimension in elements
    const float *pos;       // EPI_CONVOUT: positions [100][ldo]
    const int2 *chunk_tok;  // EPI_CONVOUT: per chunk {first packed row, rows}
    // A_CONV_S2 only: the m-tiles to compute, each chunk * 256 + tile within
    // the chunk; a tile is tile_t output time steps x all output frequencies.
    const int *tile_list;
    int rows_per_chunk;     // output rows of one chunk (T_out * F_out)
    int tile_t;             // output time steps per 128-row tile
};

template <int BN>
struct GemmCfg {
    static constexpr int BM = 128, BK = 64;
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES_RAW = (216 * 1024) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr uint32_t TMEM_COLS = 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32, 256]");
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
};

template <int EPI>
__device__ __forceinline__ void epilogue_store(const GemmArgs &a, int row, int col,
                                               const uint32_t (&r)[32])
{
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
    if constexpr (EPI == EPI_CONVOUT_F32) {
        const int chunk = row / 100, t = row - chunk * 100;
        const int2 ct = a.chunk_tok[chunk];
        if (t >= ct.y) return;
        float *dst = reinterpret_cast<float *>(a.out) + (size_t)(ct.x + t) * a.ldo + col;
        const float *p = a.pos + (size_t)t * a.ldo + col;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            float4 pp = *reinterpret_cast<const float4 *>(p + i);
            float4 o = make_float4(v[i] + pp.x, v[i + 1] + pp.y, v[i + 2] + pp.z, v[i + 3] + pp.w);
            *reinterpret_cast<float4 *>(dst + i) = o;
        }
        return;
    } else {
        const float *b = a.bias + col;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            float4 bb = *reinterpret_cast<const float4 *>(b + i);
            v[i] += bb.x;
            v[i + 1] += bb.y;
            v[i + 2] += bb.z;
            v[i + 3] += bb.w;
        }
        if constexpr (EPI == EPI_BF16 || EPI == EPI_GELU_BF16) {
            if constexpr (EPI == EPI_GELU_BF16) {
#pragma unroll
                for (int i = 0; i < 32; i++) v[i] = gelu_erf(v[i]);
            }
            bf16 *dst = reinterpret_cast<bf16 *>(a.out) + (size_t)row * a.ldo + col;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
                uint4 q = make_uint4(pack_bf16x2(v[i], v[i + 1]), pack_bf16x2(v[i + 2], v[i + 3]),
                                     pack_bf16x2(v[i + 4], v[i + 5]), pack_bf16x2(v[i + 6], v[i + 7]));
                *reinterpret_cast<uint4 *>(dst + i) = q;
            }
        } else if constexpr (EPI == EPI_RESID_F32) {
            float *dst = reinterpret_cast<float *>(a.out) + (size_t)row * a.ldo + col;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 x = *reinterpret_cast<float4 *>(dst + i);
                x.x += v[i];
                x.y += v[i + 1];
                x.z += v[i + 2];
                x.w += v[i + 3];
                *reinterpret_cast<float4 *>(dst + i) = x;
            }
        } else if constexpr (EPI == EPI_F32) {
            float *dst = reinterpret_cast<float *>(a.out) + (size_t)row * a.ldo + col;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
}

template <int BN, int EPI, int AMODE = A_PLAIN>
__global__ void __launch_bounds__(GemmCfg<BN>::THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs args)
{
    using C = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], C::EPI_WARPS);
        }
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_tiles = args.m_tiles * args.n_tiles;
    const int num_kb = args.K / C::BK;

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mt = tile % args.m_tiles, nt = tile / args.m_tiles;
                int chunk = 0, t0 = 0;
                if constexpr (AMODE == A_CONV_S2) {
                    const int item = args.tile_list[mt];
                    chunk = item >> 8;
                    t0 = (item & 255) * args.tile_t;
                }
                for (int kb = 0; kb < num_kb; kb++) {
                    if (!mbar_wait(&empty[s], ph ^ 1, args.err)) { ok = false; break; }
                    uint8_t *st = smem + s * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                    if constexpr (AMODE == A_CONV_S2) {
                        // input pixels (2 t + kt - 1, 2 f + kf - 1) of the tile's outputs;
                        // the map's traversal stride 2 on f and t does the striding
                        const int tap = kb >> 3, kf = tap / 3, kt = tap - 3 * kf;
                        tma_load_4d(&tmA, &full[s], st, (kb & 7) * 64, kf - 1, 2 * t0 + kt - 1, chunk);
                    } else {
                        tma_load_2d(&tmA, &full[s], st, kb * C::BK, mt * C::BM);
                    }
                    tma_load_2d(&tmB, &full[s], st + C::A_BYTES, kb * C::BK, nt * BN);
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, BN);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!mbar_wait(&tempty[acc], aph ^ 1, args.err)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                for (int kb = 0; kb < num_kb; kb++) {
                    if (!mbar_wait(&full[s], ph, args.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < C::BK / 16; k++)
                        mma_bf16(d, sw128_desc(a_addr + k * 32), sw128_desc(b_addr + k * 32), idesc,
                                 (kb | k) != 0);
                    mma_commit(&empty[s]);
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(&tfull[acc]);
            }
        }
    } else {
        const int q = warp & 3;             // this warp may read TMEM lanes 32q .. 32q+31
        const int half = (warp - 2) >> 2;   // which of the two warps on this quarter
        int it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            if (!mbar_wait(&tfull[acc], aph, args.err)) break;
            tc_fence_after();
            const int mt = tile % args.m_tiles, nt = tile / args.m_tiles;
            int row = mt * C::BM + q * 32 + lane;
            bool row_ok = row < args.M;
            if constexpr (AMODE == A_CONV_S2) {
                const int item = args.tile_list[mt];
                const int r_in_chunk = (item & 255) * C::BM + q * 32 + lane;
                row_ok = r_in_chunk < args.rows_per_chunk;
                row = (item >> 8) * args.rows_per_chunk + r_in_chunk;
            }
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            if constexpr (EPI == EPI_SWIGLU_BF16) {
#pragma unroll 1
                for (int c0 = 64 * half; c0 < BN; c0 += 128) {
                    uint32_t g[32], u[32];
                    tmem_ld32(tbase + c0, g);
                    tmem_ld32(tbase + c0 + 32, u);
                    tmem_ld_wait();
                    if (row_ok) {
                        const int col = nt * BN + c0;  // interleaved column of the gate block
                        const float *bg = args.bias + col, *bu = args.bias + col + 32;
                        bf16 *dst = reinterpret_cast<bf16 *>(args.out) + (size_t)row * args.ldo + col / 2;
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            float o[8];
#pragma unroll
                            for (int j = 0; j < 8; j++) {
                                float gv = __uint_as_float(g[i + j]) + bg[i + j];
                                float uv = __uint_as_float(u[i + j]) + bu[i + j];
                                o[j] = silu(gv) * uv;
                            }
                            uint4 qv = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                                  pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
                            *reinterpret_cast<uint4 *>(dst + i) = qv;
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int c0 = 32 * half; c0 < BN; c0 += 64) {
                    uint32_t r[32];
                    tmem_ld32(tbase + c0, r);
                    tmem_ld_wait();
                    if (row_ok) epilogue_store<EPI>(args, row, nt * BN + c0, r);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace moss
