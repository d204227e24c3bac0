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
// each quarter and split the tile's 64-column groups between them.
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
    // bf16 outputs only: when nonzero, each value v is also written as the pair
    // hi = bf16(v) at column c and lo = bf16(v - hi) at column c + split_off,
    // so that a following GEMM over [hi | lo] x [W | W] sees v to ~16 bits.
    int split_off;
    // 4-bit B only: 64-wide k blocks of the stored matrix; the GEMM's k block
    // kb reads stored block kb % kq_blocks (a [hi | lo] operand against [W | W]
    // stores W once)
    int kq_blocks;
    // e4m3 operands only: out = acc * row_scale[m] * col_scale[n] + bias ...
    const float *row_scale, *col_scale;
    // NVFP4 operands only (fp4.cuh): the block-scale atoms of A and B
    const uint8_t *sfa, *sfb;
};

// Each epilogue warp stages 32 rows x 128 B in shared memory (16-byte
// chunks swizzled by row) so that global stores go out as whole 128-byte
// lines, 4 or 8 rows per warp instruction, instead of one 16-byte piece per
// row.
static constexpr uint32_t EPI_STAGE_BYTES = 32 * 128;
static constexpr size_t SMEM_LIMIT = 227 * 1024;

template <int BN>
struct GemmCfg {
    static constexpr int BM = 128, BK = 64;
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t STAGING = EPI_WARPS * EPI_STAGE_BYTES;
    static constexpr int STAGES_RAW = (int)((SMEM_LIMIT - 1024 - 256 - STAGING) / STAGE_BYTES);
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr uint32_t TMEM_COLS = 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + STAGING + 256;
    static_assert(SMEM <= SMEM_LIMIT, "shared memory budget");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32, 256]");
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
};


__device__ __forceinline__ uint4 *stage_at(uint8_t *base, int row, int chunk)
{
    return reinterpret_cast<uint4 *>(base + row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ float4 ld_f4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

// Drain the accumulator columns [c0 of this warp's groups] of one tile for the
// 32 rows of this warp's TMEM lane quarter.  my_row / my_ok / my_aux describe
// the output row of this lane's tile row (aux: position index for conv_out);
// col0 is the tile's first output column in the interleaved/GEMM space.
template <int BN, int EPI, int NHALF = 2>
__device__ __forceinline__ void drain_tile(const GemmArgs &a, uint32_t tbase, int half, int lane, uint8_t *stage,
                                           int my_row, bool my_ok, int my_aux, int col0)
{
    constexpr int NG = (BN + 63) / 64;
#pragma unroll 1
    for (int g = half; g < NG; g += NHALF) {
        const int c0 = g * 64;
        // 64 columns, or the last group's rest: 32 (BN = 160) or 48 (BN = 240)
        constexpr int REST = BN % 64;
        static_assert(REST == 0 || REST == 32 || REST == 48, "BN % 64 must be 0, 32 or 48");
        const int nc = BN - c0 < 64 ? REST : 64;
        uint32_t r[64];
        tmem_ld32(tbase + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        if (nc == 64) tmem_ld32(tbase + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        if (REST == 48 && nc == 48) tmem_ld16(tbase + c0 + 32, &r[32]);
        tmem_ld_wait();
        if constexpr (EPI == EPI_SWIGLU_BF16 || EPI == EPI_BF16 || EPI == EPI_GELU_BF16) {
            // values in place (fp32 bits in r), then one or two bf16 passes
            int nv;  // values of this lane's row in this group
            if constexpr (EPI == EPI_SWIGLU_BF16) {
                // r[0..31] gate, r[32..63] up -> 32 outputs
                const float *bg = a.bias + col0 + c0, *bu = bg + 32;
#pragma unroll
                for (int j = 0; j < 32; j++) {
                    const float gv = __uint_as_float(r[j]) + bg[j];
                    const float uv = __uint_as_float(r[32 + j]) + bu[j];
                    r[j] = __float_as_uint(silu(gv) * uv);
                }
                nv = 32;
            } else {
                const float *b = a.bias + col0 + c0;
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    if (q * 8 < nc) {
                        const float4 b0 = ld_f4(b + 8 * q), b1 = ld_f4(b + 8 * q + 4);
                        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                        for (int j = 0; j < 8; j += 2) {
                            float2 o = __fadd2_rn(make_float2(__uint_as_float(r[8 * q + j]), __uint_as_float(r[8 * q + j + 1])),
                                                  make_float2(bb[j], bb[j + 1]));
                            if constexpr (EPI == EPI_GELU_BF16) o = gelu2(o);
                            r[8 * q + j] = __float_as_uint(o.x);
                            r[8 * q + j + 1] = __float_as_uint(o.y);
                        }
                    }
                }
                nv = nc;
            }
            const int ocol = EPI == EPI_SWIGLU_BF16 ? (col0 + c0) / 2 : col0 + c0;
            const int parts = a.split_off ? 2 : 1;
#pragma unroll 1
            for (int part = 0; part < parts; part++) {
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    if (q * 8 < nv) {
                        uint32_t w[4];
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const float x0 = __uint_as_float(r[8 * q + 2 * j]), x1 = __uint_as_float(r[8 * q + 2 * j + 1]);
                            if (part == 0) {
                                w[j] = pack_bf16x2(x0, x1);
                            } else {
                                const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
                                w[j] = pack_bf16x2(x0 - __low2float(hi), x1 - __high2float(hi));
                            }
                        }
                        *stage_at(stage, lane, q) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                __syncwarp();
                bf16 *out = reinterpret_cast<bf16 *>(a.out) + ocol + part * a.split_off;
                if (nv > 32) {  // 8 lanes per 128-byte row (6 of them for 48 values), 4 rows per instruction
#pragma unroll
                    for (int it = 0; it < 8; it++) {
                        const int row = it * 4 + (lane >> 3), ch = lane & 7;
                        const int grow = __shfl_sync(0xffffffffu, my_row, row);
                        const bool ok = __shfl_sync(0xffffffffu, (int)my_ok, row);
                        const uint4 v = *stage_at(stage, row, ch);
                        if (ok && ch * 8 < nv) *reinterpret_cast<uint4 *>(out + (size_t)grow * a.ldo + ch * 8) = v;
                    }
                } else {  // 32 values: 4 lanes per 64-byte row, 8 rows per instruction
#pragma unroll
                    for (int it = 0; it < 4; it++) {
                        const int row = it * 8 + (lane >> 2), ch = lane & 3;
                        const int grow = __shfl_sync(0xffffffffu, my_row, row);
                        const bool ok = __shfl_sync(0xffffffffu, (int)my_ok, row);
                        const uint4 v = *stage_at(stage, row, ch);
                        if (ok) *reinterpret_cast<uint4 *>(out + (size_t)grow * a.ldo + ch * 8) = v;
                    }
                }
                __syncwarp();
            }
        } else {
            static_assert(REST != 48, "fp32 epilogues take BN % 64 of 0 or 32");
            // fp32 results, 32 columns (128 B per row) at a time
#pragma unroll
            for (int hh = 0; hh < 2; hh++) {
                if (hh * 32 < nc) {
                    const int cc = c0 + 32 * hh;
#pragma unroll
                    for (int q = 0; q < 8; q++) {
                        float4 v = make_float4(__uint_as_float(r[32 * hh + 4 * q]), __uint_as_float(r[32 * hh + 4 * q + 1]),
                                               __uint_as_float(r[32 * hh + 4 * q + 2]), __uint_as_float(r[32 * hh + 4 * q + 3]));
                        if constexpr (EPI != EPI_CONVOUT_F32) {
                            const float4 bb = ld_f4(a.bias + col0 + cc + 4 * q);
                            v.x += bb.x;
                            v.y += bb.y;
                            v.z += bb.z;
                            v.w += bb.w;
                        }
                        *reinterpret_cast<float4 *>(stage_at(stage, lane, q)) = v;
                    }
                    __syncwarp();
                    float *out = reinterpret_cast<float *>(a.out) + col0 + cc;
                    // all loads of the pass first (residual or positions), then the stores
                    float4 add[8];
                    float *dst[8];
                    bool okv[8];
#pragma unroll
                    for (int it = 0; it < 8; it++) {
                        const int row = it * 4 + (lane >> 3), ch = lane & 7;
                        const int grow = __shfl_sync(0xffffffffu, my_row, row);
                        okv[it] = __shfl_sync(0xffffffffu, (int)my_ok, row) != 0;
                        int t = 0;
                        if constexpr (EPI == EPI_CONVOUT_F32) t = __shfl_sync(0xffffffffu, my_aux, row);
                        dst[it] = out + (size_t)grow * a.ldo + ch * 4;
                        add[it] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if constexpr (EPI == EPI_RESID_F32) {
                            if (okv[it]) add[it] = ld_f4(dst[it]);
                        } else if constexpr (EPI == EPI_CONVOUT_F32) {
                            if (okv[it]) add[it] = ld_f4(a.pos + (size_t)t * a.ldo + col0 + cc + ch * 4);
                        }
                    }
#pragma unroll
                    for (int it = 0; it < 8; it++) {
                        const int row = it * 4 + (lane >> 3), ch = lane & 7;
                        float4 v = *reinterpret_cast<const float4 *>(stage_at(stage, row, ch));
                        v.x += add[it].x;
                        v.y += add[it].y;
                        v.z += add[it].z;
                        v.w += add[it].w;
                        if (okv[it]) *reinterpret_cast<float4 *>(dst[it]) = v;
                    }
                    __syncwarp();
                }
            }
        }
    }
}

// Output through the bulk-async (TMA) unit, for plain row-major outputs:
// the 32-row slab of this warp starts at output row `row0`.  bf16 outputs
// leave in boxes of 32 rows x 64 columns (tma_store_2d); fp32 outputs in
// boxes of 32 rows x 32 columns, stored (EPI_F32) or added to the residual
// stream in L2 (EPI_RESID_F32, tma_reduce_add_2d: X + (acc + bias), the same
// single rounding as a load-add-store, with no load latency in the warp).
// Boxes are staged in `nbuf` 4 KB buffers used in turn (1024-byte aligned,
// EPI_STAGE_BYTES apart); a buffer is rewritten only after the boxes in
// flight have been read out of shared memory.
template <int BN, int EPI, int NHALF = 2, bool SCALED = false>
__device__ __forceinline__ void drain_tile_tma(const GemmArgs &a, const CUtensorMap *tmC, uint32_t tbase, int half,
                                               int lane, uint8_t *stage_base, int nbuf, int row0, int col0)
{
    static_assert(!SCALED || EPI == EPI_BF16 || EPI == EPI_GELU_BF16, "scaled operands: bf16 outputs");
    // e4m3 operands: this lane's row scale (its row of the slab)
    const float rs = SCALED && row0 + lane < a.M ? a.row_scale[row0 + lane] : 0.0f;
    constexpr bool F32_OUT = EPI == EPI_RESID_F32 || EPI == EPI_F32;
    // bf16 boxes are 64 columns wide; fp32 boxes 32, so fp32 tiles may end
    // in a 32-column group (BN = 160: groups of 64, 64 and 32)
    static_assert(BN % 64 == 0 || (F32_OUT && BN % 64 == 32), "TMA output needs whole boxes");
    static_assert(EPI == EPI_BF16 || EPI == EPI_GELU_BF16 || F32_OUT, "epilogue");
    constexpr int NG = (BN + 63) / 64;
    const bool live = row0 < a.M;  // whole slab outside the output: nothing to write
    // boxes of the previous tile may still be reading the staging buffer
    if (lane == 0) bulk_wait_read();
    int bi = 0;  // next staging buffer
    // the buffer for the next box; waits for the earlier boxes' reads when the ring wraps
    auto next_stage = [&]() -> uint8_t * {
        if (bi == nbuf) {
            bi = 0;
            if (lane == 0) bulk_wait_read();
        }
        __syncwarp();
        return stage_base + (bi++) * EPI_STAGE_BYTES;
    };
#pragma unroll 1
    for (int g = half; g < NG; g += NHALF) {
        const int c0 = g * 64;
        const int nh = BN - c0 < 64 ? 1 : 2;  // 32-column halves in this group
        uint32_t r[64];
        tmem_ld32(tbase + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        if (nh == 2) tmem_ld32(tbase + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_ld_wait();
        const float *b = a.bias + col0 + c0;
        if constexpr (EPI == EPI_BF16 || EPI == EPI_GELU_BF16) {
#pragma unroll
            for (int q = 0; q < 16; q++) {
                const float4 bb = ld_f4(b + 4 * q);
                float2 v0 = make_float2(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]));
                float2 v1 = make_float2(__uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
                if constexpr (SCALED) {
                    // (acc * row scale) * column scale + bias
                    const float4 cs = ld_f4(a.col_scale + col0 + c0 + 4 * q);
                    v0 = __ffma2_rn(__fmul2_rn(v0, make_float2(rs, rs)), make_float2(cs.x, cs.y), make_float2(bb.x, bb.y));
                    v1 = __ffma2_rn(__fmul2_rn(v1, make_float2(rs, rs)), make_float2(cs.z, cs.w), make_float2(bb.z, bb.w));
                } else {
                    v0 = __fadd2_rn(v0, make_float2(bb.x, bb.y));
                    v1 = __fadd2_rn(v1, make_float2(bb.z, bb.w));
                }
                if constexpr (EPI == EPI_GELU_BF16) {
                    v0 = gelu2(v0);
                    v1 = gelu2(v1);
                }
                r[4 * q] = __float_as_uint(v0.x);
                r[4 * q + 1] = __float_as_uint(v0.y);
                r[4 * q + 2] = __float_as_uint(v1.x);
                r[4 * q + 3] = __float_as_uint(v1.y);
            }
            const int parts = a.split_off ? 2 : 1;
#pragma unroll 1
            for (int part = 0; part < parts; part++) {
                uint8_t *stage = next_stage();
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const float x0 = __uint_as_float(r[8 * q + 2 * j]), x1 = __uint_as_float(r[8 * q + 2 * j + 1]);
                        if (part == 0) {
                            w[j] = pack_bf16x2(x0, x1);
                        } else {
                            const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
                            w[j] = pack_bf16x2(x0 - __low2float(hi), x1 - __high2float(hi));
                        }
                    }
                    *stage_at(stage, lane, q) = make_uint4(w[0], w[1], w[2], w[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0 && live) {
                    tma_store_2d(tmC, stage, col0 + c0 + part * a.split_off, row0);
                    bulk_commit();
                }
            }
        } else {
#pragma unroll
            for (int hh = 0; hh < 2; hh++) {
                if (hh >= nh) break;
                uint8_t *stage = next_stage();
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    const float4 bb = ld_f4(b + 32 * hh + 4 * q);
                    float2 v0 = make_float2(__uint_as_float(r[32 * hh + 4 * q]), __uint_as_float(r[32 * hh + 4 * q + 1]));
                    float2 v1 = make_float2(__uint_as_float(r[32 * hh + 4 * q + 2]), __uint_as_float(r[32 * hh + 4 * q + 3]));
                    v0 = __fadd2_rn(v0, make_float2(bb.x, bb.y));
                    v1 = __fadd2_rn(v1, make_float2(bb.z, bb.w));
                    *reinterpret_cast<float4 *>(stage_at(stage, lane, q)) = make_float4(v0.x, v0.y, v1.x, v1.y);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0 && live) {
                    if constexpr (EPI == EPI_RESID_F32)
                        tma_reduce_add_2d(tmC, stage, col0 + c0 + 32 * hh, row0);
                    else
                        tma_store_2d(tmC, stage, col0 + c0 + 32 * hh, row0);
                    bulk_commit();
                }
            }
        }
    }
}

// Output row of tile row `trow` for the plain and conv_out epilogues.
template <int EPI>
__device__ __forceinline__ void plain_row(const GemmArgs &a, int row, int &grow, bool &ok, int &aux)
{
    if constexpr (EPI == EPI_CONVOUT_F32) {
        const int chunk = row / 100, t = row - chunk * 100;
        const bool in = row < a.M;
        const int2 ct = in ? a.chunk_tok[chunk] : make_int2(0, 0);
        ok = in && t < ct.y;
        grow = ct.x + t;
        aux = t;
    } else {
        ok = row < a.M;
        grow = row;
        aux = 0;
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
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::STAGES * C::STAGE_BYTES + C::STAGING);
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
    if (threadIdx.x == 0) grid_dep_launch();

    if (warp == 0) {
        if (lane == 0) {
            grid_dep_wait();
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
        uint8_t *stage = smem + C::STAGES * C::STAGE_BYTES + (warp - 2) * EPI_STAGE_BYTES;
        grid_dep_wait();
        int it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            if (!mbar_wait(&tfull[acc], aph, args.err)) break;
            tc_fence_after();
            const int mt = tile % args.m_tiles, nt = tile / args.m_tiles;
            int grow, aux;
            bool ok;
            if constexpr (AMODE == A_CONV_S2) {
                const int item = args.tile_list[mt];
                const int r_in_chunk = (item & 255) * C::BM + q * 32 + lane;
                ok = r_in_chunk < args.rows_per_chunk;
                grow = (item >> 8) * args.rows_per_chunk + r_in_chunk;
                aux = 0;
            } else {
                plain_row<EPI>(args, mt * C::BM + q * 32 + lane, grow, ok, aux);
            }
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            drain_tile<BN, EPI>(args, tbase, half, lane, stage, grow, ok, aux, nt * BN);
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

// ---------------------------------------------------------------------------
// The same GEMM on CTA pairs (cluster of 2, tcgen05 cta_group::2).
//
// A pair computes a 256 x BN output tile: each CTA loads its own 128 rows of
// A and its own half of B's rows per 64-wide k-block (no multicast), and the
// even CTA's MMA thread issues M = 256 MMAs that read both CTAs' shared
// memory and write each CTA's 128 accumulator rows into that CTA's TMEM.  Per
// CTA a stage is 16 KB of A plus BN*64 B of B, and each CTA streams half the
// B traffic of the single-CTA kernel.  A 320-wide tile (N = 1280 in four)
// is two MMAs of N = 160 per k-step; the B rows of MMA j are split between
// the CTAs as rows [j*160, j*160+80) and [j*160+80, j*160+160).
//  - full[s] lives in the even CTA; both producers arrive on it (count 2) and
//    both CTAs' TMA bytes complete on it.
//  - empty[s] and tfull[acc] live in each CTA; the even CTA's MMA thread
//    commits once to its own and once to the odd CTA's barrier.
//  - tempty[acc] lives in the even CTA; all 16 epilogue warps of the pair
//    arrive on it.
// RING: every CTA pair computes at most one tile (the launch has no more
// tiles than pairs), so the epilogue always stages its output boxes in the
// idle stage ring and the separate staging area is left out: the room goes
// to the pipeline (320-wide tiles get three stages of two k sub-blocks).
template <int BN, int KSUB = 1, int BQ = 0, int RING = 0>
struct Gemm2Cfg {
    // A stage holds KSUB k sub-blocks of 64 (one 128-byte swizzle atom each):
    // larger stages halve the stage hand-offs between the producer, the MMA
    // lane and the barriers, which measurably idle the tensor pipe.
    static constexpr int BM = 128, BK = 64 * KSUB;  // rows per CTA; the pair covers 256
    // a multiple of 4 (the TMEM lane quarters); 8 measured faster than 4 on
    // the layer GEMMs (FC1 45 vs 48-50 us, out-proj 21.5 vs 24.5-25 us)
    static constexpr int EPI_WARPS = 8;
    // 4-bit B (BQ): two converter warps expand each stage's codes to bf16
    // (384 threads leave the epilogue its registers: with four, it spilled)
    static constexpr int CONV_WARPS = BQ ? 2 : 0;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS + 32 * CONV_WARPS;
    // Tiles wider than one MMA (BN = 320) are two MMAs of BN/2 per k-step.
    static constexpr int NSUB = BN > 256 ? 2 : 1;
    static constexpr int NS = BN / NSUB;                        // N of one MMA instruction
    static constexpr uint32_t B_SUB_BYTES = (NS / 2) * 64 * 2;  // this CTA's half of one MMA's B, one k sub-block
    static constexpr uint32_t A_SUB = BM * 64 * 2;              // this CTA's A rows, one k sub-block
    static constexpr uint32_t A_BYTES = KSUB * A_SUB;
    static constexpr uint32_t B_KS = NSUB * B_SUB_BYTES;        // B bytes of one k sub-block
    static constexpr uint32_t B_BYTES = KSUB * B_KS;
    // BQ: the codes of this CTA's B rows (32 bytes per row per 64-wide k
    // block, two per byte, low nibble first) and their group scales (fp32),
    // after the bf16 B they expand into.  Every TMA destination starts on a
    // 128-byte boundary (the scale boxes of NS/2 rows are padded to it).
    static constexpr uint32_t RAW_SUB = (NS / 2) * 32;
    static constexpr uint32_t SC_BOX = (NS / 2) * 4;                   // bytes one scale box brings
    static constexpr uint32_t SC_SUB = (SC_BOX + 127) / 128 * 128;     // its slot
    static constexpr uint32_t RAW_OFF = A_BYTES + B_BYTES;
    static constexpr uint32_t SC_OFF = RAW_OFF + NSUB * RAW_SUB;
    static constexpr uint32_t Q_TX = BQ ? NSUB * (RAW_SUB + SC_BOX) : 0;  // bytes completing on rawfull[s]
    static constexpr uint32_t Q_BYTES = BQ ? NSUB * (RAW_SUB + SC_SUB) : 0;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + (Q_BYTES + 1023) / 1024 * 1024;
    static_assert(RAW_OFF % 128 == 0 && SC_OFF % 128 == 0 && RAW_SUB % 128 == 0 && SC_SUB % 128 == 0,
                  "TMA destinations on 128-byte boundaries");
    // bytes each CTA's TMA completes on the pair's full barrier per stage
    static constexpr uint32_t FULL_TX = BQ ? A_BYTES : A_BYTES + B_BYTES;
    static constexpr uint32_t STAGING = RING ? 0 : EPI_WARPS * EPI_STAGE_BYTES;
    static constexpr int STAGES_RAW = (int)((SMEM_LIMIT - 1024 - 256 - STAGING) / STAGE_BYTES);
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int ACC = 2 * BN <= 512 ? 2 : 1;  // TMEM accumulators (double buffer when they fit)
    static constexpr uint32_t TMEM_COLS = ACC * BN <= 128 ? 128 : ACC * BN <= 256 ? 256 : 512;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + STAGING + 256;
    static_assert(SMEM <= SMEM_LIMIT, "shared memory budget");
    static_assert(STAGES >= 2, "at least two pipeline stages");
    static_assert(KSUB == 1 || KSUB == 2, "k sub-blocks per stage");
    static_assert(BN % 16 == 0 && BN >= 64 && BN <= 320, "BN must be a multiple of 16 in [64, 320]");
    static_assert(NS % 16 == 0 && NS <= 256, "MMA N");
    static_assert(B_SUB_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
    static_assert(!BQ || KSUB == 1, "4-bit B: one k sub-block per stage");
    static_assert(3 * STAGES * 8 + 2 * 16 + 4 <= 256, "barriers fit their area");
};

// Tile t of the pair kernel.  Plain GEMMs walk row blocks first (pairs that
// run together share a column block of the weights).  The implicit convs
// walk column blocks first: their input (the previous conv's activations) is
// far larger than L2, and the two 240-wide column blocks of a row block then
// read its input slab at the same time, once from DRAM.
template <int AMODE>
__device__ __forceinline__ void pair_tile(int tile, const GemmArgs &a, int &mt, int &nt)
{
    if constexpr (AMODE == A_CONV_S2) {
        mt = tile / a.n_tiles;
        nt = tile - mt * a.n_tiles;
    } else {
        mt = tile % a.m_tiles;
        nt = tile / a.m_tiles;
    }
}

// Expands one stage's 4-bit B codes into the bf16 B tiles the MMA reads
// (K-major, 128-byte swizzle), for the CTA's NSUB x NS/2 rows.  A value is
// bf16(fp32(q) * s): the code u = q + 8 becomes q exactly in fp32 as
// (2^23 + u) - (2^23 + 8) (u placed in the low bits of 2^23's significand),
// is scaled in fp32 and rounded to bf16 once.  Converter thread ct takes whole
// rows ct, ct + 64, ...: two 16-byte loads of codes, one scale, eight 16-byte
// stores (the 8 threads of a store wavefront write 8 consecutive rows, whose
// swizzled chunk positions differ).
template <class C>
__device__ __forceinline__ void expand_q4(uint8_t *stage, int ct)
{
    constexpr int NT = C::CONV_WARPS * 32;
    constexpr int ROWS = C::NS / 2;
    const float2 bias = make_float2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
#pragma unroll 1
    for (int rr = ct; rr < C::NSUB * ROWS; rr += NT) {
        const int j = rr / ROWS, r = rr - j * ROWS;
        const uint4 *src = reinterpret_cast<const uint4 *>(stage + C::RAW_OFF + j * C::RAW_SUB + r * 32);
        const uint4 c0 = src[0], c1 = src[1];
        const float sc = *reinterpret_cast<const float *>(stage + C::SC_OFF + j * C::SC_SUB + r * 4);
        const float2 s2 = make_float2(sc, sc);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint8_t *row = stage + C::A_BYTES + j * C::B_SUB_BYTES + r * 128;
#pragma unroll
        for (int c = 0; c < 8; c++) {
            // chunk c: k = 8 c .. 8 c + 7; byte b holds k = 8 c + 2 b (low nibble), 8 c + 2 b + 1
            const uint32_t lo = words[c] & 0x0F0F0F0Fu, hi = (words[c] >> 4) & 0x0F0F0F0Fu;
            uint32_t o[4];
#pragma unroll
            for (int b = 0; b < 4; b++) {
                const float2 m = make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650u + b)),
                                             __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650u + b)));
                const float2 v = __fmul2_rn(__fadd2_rn(m, bias), s2);
                o[b] = pack_bf16x2(v.x, v.y);
            }
            *reinterpret_cast<uint4 *>(row + ((c ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// Up to four 4-bit matrices to expand in one launch: codes [n][kq/2], scales
// [kq/128][n] -> bf16 rows out [n][reps * kq] (the row's kq values repeated
// reps times along k).
struct Q4Job {
    const uint8_t *codes;
    const float *scales;
    bf16 *out;
    int n, kq, reps;
    long long first;  // first item of this job (items: 32 values of one row)
};
struct Q4Jobs {
    Q4Job j[4];
    int count;
    long long items;
};

// Expands the jobs' matrices with the arithmetic of expand_q4.  Thread i
// takes 32 consecutive k of one row (16 bytes of codes, one scale) and writes
// 64 bytes per repeat.  The outputs are scratch that earlier kernels may
// still read: the writes wait for them.
__global__ void __launch_bounds__(256) q4_expand_kernel(const __grid_constant__ Q4Jobs jobs)
{
    grid_dep_wait();
    grid_dep_launch();
    const float2 bias = make_float2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < jobs.items;
         i += (long long)gridDim.x * blockDim.x) {
        int jb = 0;
        while (jb + 1 < jobs.count && i >= jobs.j[jb + 1].first) jb++;
        const Q4Job &J = jobs.j[jb];
        const long long li = i - J.first;
        const int per_row = J.kq / 32;
        const int r = (int)(li / per_row), k0 = (int)(li - (long long)r * per_row) * 32;
        const uint4 c = *reinterpret_cast<const uint4 *>(J.codes + (size_t)r * (J.kq / 2) + k0 / 2);
        const float sc = J.scales[(size_t)(k0 / 128) * J.n + r];
        const float2 s2 = make_float2(sc, sc);
        const uint32_t words[4] = {c.x, c.y, c.z, c.w};
        uint4 o[4];
#pragma unroll
        for (int w = 0; w < 4; w++) {
            const uint32_t lo = words[w] & 0x0F0F0F0Fu, hi = (words[w] >> 4) & 0x0F0F0F0Fu;
            uint32_t v[4];
#pragma unroll
            for (int b = 0; b < 4; b++) {
                const float2 m = make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7650u + b)),
                                             __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7650u + b)));
                const float2 x = __fmul2_rn(__fadd2_rn(m, bias), s2);
                v[b] = pack_bf16x2(x.x, x.y);
            }
            o[w] = make_uint4(v[0], v[1], v[2], v[3]);
        }
        for (int rep = 0; rep < J.reps; rep++) {
            uint4 *dst = reinterpret_cast<uint4 *>(J.out + (size_t)r * J.reps * J.kq + (size_t)rep * J.kq + k0);
#pragma unroll
            for (int w = 0; w < 4; w++) dst[w] = o[w];
        }
    }
}


// F8: A and B are e4m3 (one byte per element, so a 128-byte swizzled row holds
// 128 k, and the stages' byte sizes are the bf16 ones), multiplied with
// kind::f8f6f4; the epilogue scales by the row and column scales.
template <int BN, int EPI, int AMODE = A_PLAIN, int KSUB = 1, int BQ = 0, int F8 = 0, int RING = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm2Cfg<BN, KSUB, BQ, RING>::THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmS,
                    const GemmArgs args)
{
    using C = Gemm2Cfg<BN, KSUB, BQ, RING>;
    static_assert(!BQ || AMODE == A_PLAIN, "4-bit B for plain GEMMs");
    static_assert(!F8 || (AMODE == A_PLAIN && !BQ), "e4m3 operands for plain GEMMs");
    constexpr int EK = F8 ? 128 : 64;  // k elements per 128-byte row
    // plain row-major outputs leave through TMA boxes (tmC); the conv and
    // conv_out row mappings and SwiGLU keep per-row stores
    constexpr bool TMA_OUT = AMODE == A_PLAIN &&
                             ((BN % 64 == 0 && (EPI == EPI_BF16 || EPI == EPI_GELU_BF16 || EPI == EPI_RESID_F32 ||
                                                EPI == EPI_F32)) ||
                              (BN % 64 == 32 && (EPI == EPI_RESID_F32 || EPI == EPI_F32)));
    static_assert(!RING || TMA_OUT, "only the TMA epilogue stages in the ring");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::STAGES * C::STAGE_BYTES + C::STAGING);
    uint64_t *empty = full + C::STAGES;
    uint64_t *rawfull = empty + C::STAGES;  // BQ: this CTA's codes and scales of stage s have landed
    uint64_t *tfull = rawfull + C::STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; s++) {
            // both producers arrive (with their TMA bytes); with 4-bit B also
            // one converter thread of each CTA once its bf16 B is in place
            mbar_init(&full[s], BQ ? 4 : 2);
            mbar_init(&empty[s], 1);
            mbar_init(&rawfull[s], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 2 * C::EPI_WARPS);
        }
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if constexpr (TMA_OUT) prefetch_tmap(&tmC);
        if constexpr (BQ) prefetch_tmap(&tmS);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_tiles = args.m_tiles * args.n_tiles;  // m_tiles counts 256-row pair tiles
    const int num_kb = args.K / (EK * KSUB);
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    // TMEM is held by every started CTA of this grid: the next kernel may start
    if (threadIdx.x == 0) grid_dep_launch();

    if (warp == 0) {
        if (lane == 0) {
            auto load_b = [&](uint8_t *st, uint32_t fb, int kb, int nt, int s) {
                if constexpr (BQ) {
                    // this CTA's codes and scales, completing on its own rawfull[s]
                    const int kq = kb % args.kq_blocks;
                    mbar_arrive_expect_tx(&rawfull[s], C::Q_TX);
#pragma unroll
                    for (int j = 0; j < C::NSUB; j++) {
                        const int row0 = nt * BN + j * C::NS + (int)rank * (C::NS / 2);
                        tma_load_2d(&tmB, &rawfull[s], st + C::RAW_OFF + j * C::RAW_SUB, kq * 32, row0);
                        tma_load_2d(&tmS, &rawfull[s], st + C::SC_OFF + j * C::SC_SUB, row0, kq >> 1);
                    }
                } else {
#pragma unroll
                    for (int ks = 0; ks < KSUB; ks++)
#pragma unroll
                        for (int j = 0; j < C::NSUB; j++)
                            tma_load_2d_pair(&tmB, fb, st + C::A_BYTES + ks * C::B_KS + j * C::B_SUB_BYTES,
                                             (kb * KSUB + ks) * EK, nt * BN + j * C::NS + (int)rank * (C::NS / 2));
                }
            };
            // The weights do not depend on earlier kernels: the first tile's
            // first stages of B are requested before waiting for them (each
            // stage's first use needs no wait on its empty barrier).
            const int npre = pair < num_tiles ? (num_kb < C::STAGES ? num_kb : C::STAGES) : 0;
            for (int kb = 0; kb < npre; kb++) {
                const uint32_t fb = map_to_rank(smem_u32(&full[kb]), 0);
                mbar_arrive_expect_tx_remote(fb, C::FULL_TX);
                int mt0, nt0;
                pair_tile<AMODE>(pair, args, mt0, nt0);
                load_b(smem + kb * C::STAGE_BYTES, fb, kb, nt0, kb);
            }
            grid_dep_wait();
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                int mt, nt;
                pair_tile<AMODE>(tile, args, mt, nt);
                int chunk = 0, t0 = 0;
                if constexpr (AMODE == A_CONV_S2) {
                    const int item = args.tile_list[2 * mt + rank];  // padded list: -1 = no rows
                    chunk = item < 0 ? 0 : item >> 8;
                    t0 = item < 0 ? 0 : (item & 255) * args.tile_t;
                }
                for (int kb = 0; kb < num_kb; kb++) {
                    const bool pre = tile == pair && kb < npre;  // B already requested
                    uint8_t *st = smem + s * C::STAGE_BYTES;
                    const uint32_t fb = map_to_rank(smem_u32(&full[s]), 0);
                    if (!pre) {
                        if (!mbar_wait(&empty[s], ph ^ 1, args.err)) { ok = false; break; }
                        mbar_arrive_expect_tx_remote(fb, C::FULL_TX);
                    }
#pragma unroll
                    for (int ks = 0; ks < KSUB; ks++) {
                        if constexpr (AMODE == A_CONV_S2) {
                            // 64-wide k block b = tap * 8 + channel block
                            const int b = kb * KSUB + ks, tap = b >> 3, kf = tap / 3, kt = tap - 3 * kf;
                            tma_load_4d_pair(&tmA, fb, st + ks * C::A_SUB, (b & 7) * 64, kf - 1, 2 * t0 + kt - 1, chunk);
                        } else {
                            tma_load_2d_pair(&tmA, fb, st + ks * C::A_SUB, (kb * KSUB + ks) * EK, mt * 256 + (int)rank * 128);
                        }
                    }
                    if (!pre) load_b(st, fb, kb, nt, s);
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = F8 ? idesc_e4m3(256, C::NS) : idesc_bf16(256, C::NS);
            // Descriptors and barrier addresses are formed once: the issue loop
            // shares its SM sub-partition with epilogue warps, and every
            // instruction it saves brings the next MMA to the tensor pipe sooner.
            // A descriptor's start-address field is the byte address / 16, so
            // stage s and k-step k add (s * STAGE_BYTES + 32 k) / 16 to stage 0's.
            const uint64_t a_desc0 = sw128_desc(smem_u32(smem));
            const uint32_t emp0 = map_to_rank(smem_u32(&empty[0]), 0), emp1 = map_to_rank(smem_u32(&empty[0]), 1);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int it = 0;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++it) {
                const int acc = it % C::ACC;
                const uint32_t aph = (it / C::ACC) & 1;
                if (!mbar_wait(&tempty[acc], aph ^ 1, args.err)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                for (int kb = 0; kb < num_kb; kb++) {
                    // 4-bit B: the phase also publishes both CTAs' converter stores
                    const bool got = BQ ? mbar_wait_cluster(&full[s], ph, args.err) : mbar_wait(&full[s], ph, args.err);
                    if (!got) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = a_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const uint64_t bd = ad + (C::A_BYTES >> 4);
#pragma unroll
                    for (int ks = 0; ks < KSUB; ks++) {
                        // conv: the last channel block of a tap holds channels 448..479 and
                        // 32 zeros (past the 480 channels); its zero half is not multiplied
                        const int nk = (AMODE == A_CONV_S2 && ((kb * KSUB + ks) & 7) == 7) ? 2 : 4;
#pragma unroll
                        for (int k = 0; k < 4; k++)
#pragma unroll
                            for (int j = 0; j < C::NSUB; j++)
                                if (k < nk) {
                                    const uint64_t da = ad + ks * (C::A_SUB >> 4) + 2 * k;
                                    const uint64_t db = bd + ks * (C::B_KS >> 4) + j * (C::B_SUB_BYTES >> 4) + 2 * k;
                                    if constexpr (F8)
                                        mma_e4m3_pair(d + j * C::NS, da, db, idesc, (kb | ks | k) != 0);
                                    else
                                        mma_bf16_pair(d + j * C::NS, da, db, idesc, (kb | ks | k) != 0);
                                }
                    }
                    mma_commit_pair(emp0 + 8 * s);
                    mma_commit_pair(emp1 + 8 * s);
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
                if (ok) {
                    const uint32_t tb = smem_u32(&tfull[acc]);
                    mma_commit_pair(map_to_rank(tb, 0));
                    mma_commit_pair(map_to_rank(tb, 1));
                }
            }
        }
    } else if (warp < 2 + C::EPI_WARPS) {
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;  // which of the warps on this lane quarter
        uint8_t *stage = smem + C::STAGES * C::STAGE_BYTES + (warp - 2) * EPI_STAGE_BYTES;
        grid_dep_wait();
        int it = 0;
        for (int tile = pair; tile < num_tiles; tile += npairs, ++it) {
            const int acc = it % C::ACC;
            const uint32_t aph = (it / C::ACC) & 1;
            int mt, nt;
            pair_tile<AMODE>(tile, args, mt, nt);
            if constexpr (EPI == EPI_RESID_F32) {
                // the residual rows this tile adds to go to L2 while the mainloop runs
                const int row = mt * 256 + (int)rank * 128 + q * 32 + lane;
                if (half == 0 && row < args.M)
                    prefetch_l2(reinterpret_cast<const float *>(args.out) + (size_t)row * args.ldo + nt * BN, BN * 4);
            }
            if (!mbar_wait(&tfull[acc], aph, args.err)) break;
            tc_fence_after();
            int grow, aux;
            bool ok;
            if constexpr (AMODE == A_CONV_S2) {
                const int item = args.tile_list[2 * mt + rank];
                const int r_in_chunk = (item & 255) * 128 + q * 32 + lane;
                ok = item >= 0 && r_in_chunk < args.rows_per_chunk;
                grow = (item >> 8) * args.rows_per_chunk + r_in_chunk;
                aux = 0;
            } else {
                plain_row<EPI>(args, mt * 256 + (int)rank * 128 + q * 32 + lane, grow, ok, aux);
            }
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            if constexpr (TMA_OUT) {
                // On the CTA's last tile the stage ring is idle once the
                // accumulator is full (every load of this CTA has been consumed),
                // so each epilogue warp stages through its eighth of the ring and
                // keeps several boxes in flight; otherwise one 4 KB buffer.
                constexpr int RING_BUFS = (int)(C::STAGES * C::STAGE_BYTES / C::EPI_WARPS / EPI_STAGE_BYTES);
                const bool last = RING || tile + npairs >= num_tiles;
                uint8_t *stg = last ? smem + (warp - 2) * RING_BUFS * EPI_STAGE_BYTES : stage;
                drain_tile_tma<BN, EPI, C::EPI_WARPS / 4, F8 != 0>(args, &tmC, tbase, half, lane, stg,
                                                                     last ? RING_BUFS : 1,
                                                                     mt * 256 + (int)rank * 128 + q * 32, nt * BN);
            } else
                drain_tile<BN, EPI, C::EPI_WARPS / 4>(args, tbase, half, lane, stage, grow, ok, aux, nt * BN);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(map_to_rank(smem_u32(&tempty[acc]), 0));
        }
        if constexpr (TMA_OUT) {
            if (lane == 0) bulk_wait_all();  // this warp's output boxes are written before the grid ends
        }
    } else if constexpr (BQ) {
        // converters: stage s's codes -> bf16 B, then one arrive on the pair's
        // full[s].  The codes are the weights (no earlier kernel writes them),
        // so there is no wait on earlier grids.  A stage's B is rewritten only
        // after its next codes land, which the producer requests only once the
        // MMAs that read the stage have completed.
        const int ct = threadIdx.x - 32 * (2 + C::EPI_WARPS);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
            for (int kb = 0; kb < num_kb; kb++) {
                if (!mbar_wait(&rawfull[s], ph, args.err)) { ok = false; break; }
                uint8_t *st = smem + s * C::STAGE_BYTES;
                expand_q4<C>(st, ct);
                fence_async_smem();  // the generic-proxy stores are seen by the MMA's reads
                named_bar_sync(1, C::CONV_WARPS * 32);
                if (ct == 0) mbar_arrive_release_cluster(map_to_rank(smem_u32(&full[s]), 0));
                if (++s == C::STAGES) { s = 0; ph ^= 1; }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its partner may still touch its memory
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
}

}  // namespace moss
