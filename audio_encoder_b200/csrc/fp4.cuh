// NVFP4 GEMMs on the block-scaled FP4 tensor cores (page "Ossicle-4B",
// section "Quantized: NVFP4 and INT4 in vLLM": NVFP4 weights and activations
// for the audio encoder, run by Blackwell's native FP4 kernels).
//
// NVFP4 operand: E2M1 elements packed two per byte (even k in the low
// nibble) in rows of K/2 bytes; one E4M3 scale per 16 consecutive elements
// along K; one fp32 factor g per weight matrix and per activation row,
// applied in the epilogue:
//   out[m][n] = (sum_k (q_a s_a)[m][k] (q_w s_w)[n][k]) * g_a[m] * g_w + b[n]
// The block scales live in global memory in the tensor cores' own order:
// 512-byte atoms of 128 rows x 64 k (four scales per row), row r of the atom
// at byte (r % 32) * 16 + (r / 32) * 4 + (k / 16), atoms ordered [rows / 128]
// [K / 64] (k fastest), so that a stage's four atoms are one contiguous copy.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "gemm.cuh"

namespace moss {

// 1-D bulk copy global -> shared, completing on an mbarrier (both addresses
// 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory descriptor of one scale atom for tcgen05.cp: 32 rows of 16
// bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t smem_addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(128 >> 4) << 32;  // stride between 8-row core matrices
    d |= (uint64_t)1 << 46;           // descriptor version (sm_100); layout type 0 = no swizzle
    return d;
}

// One scale atom (32 rows x 128 bits) into TMEM lanes 0..31 of four columns,
// repeated in the other three lane quarters: lane r % 32 of every quarter,
// column r / 32, byte k / 16 -- the layout the block-scaled MMA reads.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A * B^T on E2M1 operands with E4M3 scales per 16 (M = 128, K = 64).
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem));
}

// Instruction descriptor of the block-scaled kind: A and B E2M1 (format 1 of
// the FP4 kinds), both K-major, scales E4M3 (scale format 0), scale ids 0,
// dense K = 64; the accumulator is fp32 by definition of the kind.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N)
{
    return (1u << 7)                      // A format E2M1
           | (1u << 10)                   // B format E2M1
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

template <int BN>
struct Fp4Cfg {
    static constexpr int BM = 128;
    static constexpr int KB = 256;  // k elements per stage: one 128-byte swizzle row per operand row
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr uint32_t A_BYTES = BM * 128, B_BYTES = BN * 128;
    static constexpr uint32_t SFA_BYTES = (BM / 128) * 4 * 512, SFB_BYTES = (BN / 128) * 4 * 512;
    static constexpr uint32_t SFA_OFF = A_BYTES + B_BYTES, SFB_OFF = SFA_OFF + SFA_BYTES;
    static constexpr uint32_t STAGE_BYTES = (SFB_OFF + SFB_BYTES + 1023) / 1024 * 1024;
    static constexpr uint32_t STAGING = EPI_WARPS * EPI_STAGE_BYTES;
    static constexpr int STAGES_RAW = (int)((SMEM_LIMIT - 1024 - 256 - STAGING) / STAGE_BYTES);
    static constexpr int STAGES = STAGES_RAW > 6 ? 6 : STAGES_RAW;
    // TMEM: two accumulators of BN columns, then per stage the scale atoms
    // (four columns each: 4 for A's k steps, 4 x BN / 128 for B's)
    static constexpr uint32_t SF_COLS = 4 * 4 + 4 * 4 * (BN / 128);
    static constexpr uint32_t SF_BASE = 2 * BN;
    static_assert(SF_BASE + STAGES * SF_COLS <= 512, "TMEM budget");
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + STAGING + 256;
    static_assert(SMEM <= SMEM_LIMIT && STAGES >= 3, "shared memory budget");
    static_assert(BN == 128, "tile width (the B scales of one MMA are one atom)");
};

// The NVFP4 GEMM, one CTA per SM walking 128 x BN output tiles (row blocks
// first): warp 0 streams A and B by TMA and the stage's scale atoms by bulk
// copies onto the stage's barrier; warp 1 (one thread) moves each stage's
// atoms into TMEM (tcgen05.cp) and issues the four K = 64 MMAs into one of
// two TMEM accumulators; warps 2-9 drain the accumulator through the scaled
// TMA epilogue (acc * row_scale[m] * col_scale[n] + bias, GELU for
// EPI_GELU_BF16), with row_scale = g_a and col_scale = g_w.
template <int BN, int EPI>
__global__ void __launch_bounds__(Fp4Cfg<BN>::THREADS, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const GemmArgs args)
{
    using C = Fp4Cfg<BN>;
    static_assert(EPI == EPI_BF16 || EPI == EPI_GELU_BF16, "bf16 outputs");
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
        prefetch_tmap(&tmC);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int num_tiles = args.m_tiles * args.n_tiles;
    const int num_kb = args.K / C::KB;
    const int k64 = args.K / 64;  // scale atoms per 128 rows
    if (threadIdx.x == 0) grid_dep_launch();  // TMEM is held

    if (warp == 0) {
        if (lane == 0) {
            grid_dep_wait();
            int s = 0;
            uint32_t ph = 0, armed = 0;  // armed: stages with a load issued (drain on error)
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mt = tile % args.m_tiles, nt = tile / args.m_tiles;
                for (int kb = 0; kb < num_kb; kb++) {
                    if (!mbar_wait(&empty[s], ph ^ 1, args.err)) { ok = false; break; }
                    uint8_t *st = smem + s * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES + C::SFA_BYTES + C::SFB_BYTES);
                    tma_load_2d(&tmA, &full[s], st, kb * 128, mt * 128);
                    tma_load_2d(&tmB, &full[s], st + C::A_BYTES, kb * 128, nt * BN);
                    bulk_load(st + C::SFA_OFF, args.sfa + ((size_t)mt * k64 + 4 * kb) * 512, 2048, &full[s]);
#pragma unroll
                    for (int j = 0; j < BN / 128; j++)
                        bulk_load(st + C::SFB_OFF + j * 2048,
                                  args.sfb + ((size_t)(nt * (BN / 128) + j) * k64 + 4 * kb) * 512, 2048, &full[s]);
                    armed |= 1u << s;
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
            }
            if (!ok || *(volatile int *)args.err != 0) {
                // loads still in flight land before the CTA leaves (bounded)
                for (int i = 0; i < C::STAGES; i++) {
                    const int st = (s + i) % C::STAGES;  // oldest first
                    if (armed & (1u << st)) mbar_drain(&full[st], (st < s ? ph : ph ^ 1) & 1);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(128, BN);
            const uint64_t a_desc0 = sw128_desc(smem_u32(smem));
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int it = 0;
            int last_s = -1;  // stage and parity of the last commit (drain on error)
            uint32_t last_ph = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!mbar_wait(&tempty[acc], aph ^ 1, args.err)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                for (int kb = 0; kb < num_kb; kb++) {
                    if (!mbar_wait(&full[s], ph, args.err)) { ok = false; break; }
                    tc_fence_after();
                    uint8_t *st = smem + s * C::STAGE_BYTES;
                    const uint32_t sf = tmem_base + C::SF_BASE + s * C::SF_COLS;
                    // the stage's scale atoms into its TMEM slot: A's k step j at
                    // columns 4 j .. 4 j + 3, B's at 16 + 4 j (row r of a 128-row
                    // operand: lane r % 32, column r / 32, byte k / 16)
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        tmem_cp_sf(sf + 4 * j, sf_atom_desc(smem_u32(st + C::SFA_OFF + 512 * j)));
                        tmem_cp_sf(sf + 16 + 4 * j, sf_atom_desc(smem_u32(st + C::SFB_OFF + 512 * j)));
                    }
                    const uint64_t ad = a_desc0 + (uint64_t)((s * C::STAGE_BYTES) >> 4);
                    const uint64_t bd = ad + (C::A_BYTES >> 4);
#pragma unroll
                    for (int j = 0; j < 4; j++)  // K = 64 per MMA: 32 bytes of each 128-byte row
                        mma_nvf4(d, ad + 2 * j, bd + 2 * j, idesc, sf + 4 * j, sf + 16 + 4 * j, (kb | j) != 0);
                    mma_commit(&empty[s]);
                    last_s = s;
                    last_ph = ph;
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(&tfull[acc]);
            }
            // a wait that gave up: the MMAs already issued finish (bounded)
            // before the TMEM columns are released
            if (*(volatile int *)args.err != 0 && last_s >= 0) mbar_drain(&empty[last_s], last_ph);
        }
    } else {
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        uint8_t *stage = smem + C::STAGES * C::STAGE_BYTES + (warp - 2) * EPI_STAGE_BYTES;
        grid_dep_wait();
        int it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const int mt = tile % args.m_tiles, nt = tile / args.m_tiles;
            if (!mbar_wait(&tfull[acc], aph, args.err)) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            drain_tile_tma<BN, EPI, C::EPI_WARPS / 4, true>(args, &tmC, tbase, half, lane, stage, 1,
                                                          mt * 128 + q * 32, nt * BN);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (lane == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 512);
}

}  // namespace moss

namespace moss {

// fp32 pair -> two E2M1 codes in one byte, round to nearest even with
// saturation at +-6 (the value of `lo` in the low nibble).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// NVFP4 activation rows of 1280 (the operands of the q/k/v and fc1 GEMMs):
// with LN, the LayerNorm of the residual-stream row first (the same
// arithmetic as layernorm1280_kernel), else the row as given.  Then, per row,
// g = amax / 2688, per block of 16 s_b = e4m3(amax_b / (g * 6)) and the
// codes e2m1(x / (s_b * g)) (0 when s_b = 0), all in fp32: codes [rows][640]
// bytes, scale atoms [rows / 128][20][512] bytes (the GEMM's layout), g
// [rows].  One warp per row; lane l holds columns 128 i + 4 l .. + 3, so a
// block of 16 is four neighbouring lanes.
template <bool LN>
__global__ void __launch_bounds__(256, 4) nvf4_rows1280_kernel(const float *__restrict__ x, const float *__restrict__ gamma,
                                                           const float *__restrict__ beta, uint8_t *__restrict__ codes,
                                                           uint8_t *__restrict__ atoms, float *__restrict__ g_out,
                                                           int rows)
{
    grid_dep_wait();
    grid_dep_launch();
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float4 *xr = reinterpret_cast<const float4 *>(x + (size_t)row * 1280);
    float4 v[10];
#pragma unroll
    for (int i = 0; i < 10; i++) v[i] = xr[lane + 32 * i];
    if (LN) {
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i < 10; i++) s += v[i].x + v[i].y + v[i].z + v[i].w;
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
#pragma unroll
        for (int i = 0; i < 10; i++) {
            const float4 g = g4[lane + 32 * i], b = b4[lane + 32 * i];
            v[i].x = (v[i].x - mean) * rstd * g.x + b.x;
            v[i].y = (v[i].y - mean) * rstd * g.y + b.y;
            v[i].z = (v[i].z - mean) * rstd * g.z + b.z;
            v[i].w = (v[i].w - mean) * rstd * g.w + b.w;
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 10; i++)
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float g = amax / 2688.0f;
    if (lane == 0) g_out[row] = g;
    uint16_t *crow = reinterpret_cast<uint16_t *>(codes + (size_t)row * 640);
    uint8_t *arow = atoms + (size_t)(row >> 7) * 20 * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4;
#pragma unroll
    for (int i = 0; i < 10; i++) {
        float bmax = fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w)));
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));
        const __nv_fp8_storage_t sc = g > 0.0f ? __nv_cvt_float_to_fp8(bmax / (g * 6.0f), __NV_SATFINITE, __NV_E4M3)
                                               : (__nv_fp8_storage_t)0;
        const float sb = __half2float(__half(__nv_cvt_fp8_to_halfraw(sc, __NV_E4M3)));
        const float sg = sb * g;
        uint32_t c = 0;
        if (sb > 0.0f)
            c = e2m1x2(v[i].x / sg, v[i].y / sg) | (e2m1x2(v[i].z / sg, v[i].w / sg) << 8);
        crow[64 * i / 2 + lane] = (uint16_t)c;  // columns 128 i + 4 l .. + 3: bytes 64 i + 2 l, + 1
        const int b = 8 * i + (lane >> 2);       // block of 16 along the row
        if ((lane & 3) == 0) arow[(b >> 2) * 512 + (b & 3)] = (uint8_t)sc;
    }
}

}  // namespace moss
