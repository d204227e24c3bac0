// C ABI of the B200 audio encoder (declared in include/moss_enc.h): weight
// repacking, the device workspace, per-call chunk planning on the host, and
// the launch sequence of one forward.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <thread>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include <cuda_fp8.h>

#include "../../include/moss_enc.h"
#include "attn.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "mel.cuh"
#include "norm.cuh"
#include "stem.cuh"
#include "fp4.cuh"

using namespace moss;

namespace {

constexpr int D = 1280, DQKV = 3840, DFF = 5120, CST = 480, DOUT = 2048, DADP = 8192;
constexpr int CHUNK_FRAMES = 800, CHUNK_TOKENS = 100, CHUNK_SAMPLES = 128000, HOP = 160;
constexpr int CONV_K = 9 * 512;  // conv2/conv3 patch width: 9 taps x 480 channels padded to 512
constexpr int CONV_BN = 240;     // conv2/conv3 output channels per pair tile (480 in two)
constexpr int STEM_GROUP_DEFAULT = 32;
constexpr int C2_TILES = 50, C3_TILES = 13;  // 128-row tiles per chunk of conv2 (4 t x 32 f) / conv3 (8 t x 16 f)

// A weight matrix kept as 4-bit codes: codes [N][Kq/2] bytes (two per byte,
// low nibble first, code = q + 8) and scales [Kq/128][N] fp32 (group-major).
struct QW {
    const uint8_t *codes = nullptr;
    const float *scales = nullptr;
    int kq = 0;  // stored K (a [hi | lo] GEMM over [W | W] has K = 2 kq)
};

// A layer's weights: bf16 matrices, or (4-bit handles) their codes.
struct LayerDev {
    float *ln1_g, *ln1_b, *ln2_g, *ln2_b;
    bf16 *wqkv, *wo, *w1, *w2;
    float *bqkv, *bo, *b1, *b2;
    QW qqkv, qo, q1, q2;
    // FP8 handles: q/k/v and fc1 as e4m3 [N][K] with per-channel scales [N]
    const uint8_t *wqkv8 = nullptr, *w18 = nullptr;
    const float *sqkv = nullptr, *s1 = nullptr;
    // NVFP4 handles: q/k/v and fc1 codes, scale atoms and per-column g
    const uint8_t *wqkv4 = nullptr, *sqkv4 = nullptr, *w14 = nullptr, *s14 = nullptr;
    const float *gqkv4 = nullptr, *g14 = nullptr;
};

// ln_post, proj1, proj2 and the SwiGLU adapter: the encoder's own set, and
// one per layer tap (the cross-layer taps each have their own projector).
// A set with 4-bit matrices has qp1.codes set.
struct HeadDev {
    float *lnp_g, *lnp_b, *bp1, *bp2, *bgu, *bd;
    bf16 *wp1, *wp2, *wgu, *wd;
    QW qp1, qp2, qgu, qd;
};

struct ClipPlan {
    int64_t n, F, f_begin, f_end, c_first, c_last, tok0, ntok;
};

}  // namespace

struct moss_enc {
    moss_enc_config cfg{};
    int device = 0, num_sms = 148;
    cudaStream_t stream = nullptr;
    std::string last_error;

    // weights (one allocation; 4-bit handles keep the linear layers' codes
    // and scales in a second one)
    void *wmem = nullptr, *qmem = nullptr;
    bool q4 = false, fp8 = false, nvfp4 = false;
    uint8_t *sfa4 = nullptr;  // NVFP4 handles: the activation rows' scale atoms
    const uint4 *conv1_wt = nullptr;  // conv1 as the B operand of its GEMM (see conv1_tc_kernel)
    float *conv2_b = nullptr, *conv3_b = nullptr;
    bf16 *conv2_w = nullptr, *conv3_w = nullptr, *conv_out_w = nullptr;
    std::vector<LayerDev> layers;
    HeadDev head{};
    float *pos = nullptr;
    Mel4Tab *mel4_tab = nullptr;

    // layer taps (moss_enc_set_taps): encoder layer per tap and its head set
    void *tap_wmem = nullptr;
    std::vector<int> tap_layers;
    std::vector<HeadDev> tap_heads;

    // capacity
    int64_t max_tokens = 0, max_chunks = 0;
    int stem_group = STEM_GROUP_DEFAULT;

    // workspace (one allocation)
    void *ws = nullptr;
    float *mel_raw = nullptr;
    bf16 *c1out = nullptr, *c2out = nullptr, *c3out = nullptr;
    float *X = nullptr;
    bf16 *xn = nullptr, *qkv = nullptr, *attn = nullptr, *ffn = nullptr, *hb = nullptr, *h2 = nullptr, *gu = nullptr;
    int *gmax_ord = nullptr;
    int *err = nullptr;
    float *pcm_stage = nullptr;
    void *out_stage = nullptr;
    bf16 *qscratch = nullptr;  // 4-bit handles: one expanded weight matrix
    float *row_scale = nullptr;  // FP8 handles: the e4m3 LayerNorm rows' scales [T]

    // per-call tables: device copies and a ring of pinned host staging areas
    // (a call writes the next area once the copy that last read it has run,
    // so the host may run several calls ahead of the device)
    static constexpr int TAB_SLOTS = 4;
    size_t tab_bytes = 0;
    void *d_tab = nullptr, *h_tab = nullptr, *h_tab_ring = nullptr;
    cudaEvent_t tab_event[TAB_SLOTS] = {};
    int tab_slot = 0;

    // launches may overlap the previous kernel's tail (programmatic dependent
    // launch); MOSS_ENC_PDL=0 in the environment at create turns it off.
    // pdl_skip_once: the next launch waits for the previous kernel in full (a
    // GEMM whose B operand the previous kernel writes, since GEMMs request
    // their first B stages before waiting on earlier kernels).
    bool pdl = true, pdl_skip_once = false;

    // measurement: launch counter and optional per-launch CUDA events
    int64_t launches = 0;
    bool profiling = false;
    struct Rec {
        const char *name;
        int e0;
        double flops, bytes;
    };
    std::vector<cudaEvent_t> prof_ev;
    std::vector<Rec> prof_rec;

    // CUDA graph of the last forward request (replayed while it repeats)
    void *d_tab_graph = nullptr;
    cudaGraphExec_t graph_exec = nullptr;
    std::vector<uint8_t> graph_key;
    std::vector<uint8_t> last_key;  // the previous graphable request (run launch by launch)
    int64_t graph_launches = 0;
};

namespace {
// Counts one kernel launch and, while profiling, brackets it with events.
struct Launch {
    moss_enc *h;
    const char *name;
    double flops, bytes;
    int e0 = -1;
    Launch(moss_enc *h_, const char *name_, double flops_, double bytes_)
        : h(h_), name(name_), flops(flops_), bytes(bytes_)
    {
        h->launches++;
        if (h->profiling && h->prof_rec.size() * 2 + 2 <= h->prof_ev.size()) {
            e0 = (int)h->prof_rec.size() * 2;
            cudaEventRecord(h->prof_ev[e0], h->stream);
        }
    }
    ~Launch()
    {
        if (e0 >= 0) {
            cudaEventRecord(h->prof_ev[e0 + 1], h->stream);
            h->prof_rec.push_back(moss_enc::Rec{name, e0, flops, bytes});
        }
    }
};
}  // namespace

// ------------------------------------------------------------ small helpers

// Launch `kern` on the handle's stream.  With h->pdl the launch carries
// programmatic stream serialisation: the kernel may start while the previous
// one finishes, and waits for it (griddepcontrol.wait) before touching its
// results; every kernel launched here does so.
template <typename... KArgs, typename... Args>
static cudaError_t launch_k(moss_enc *h, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = h->stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = h->pdl && !h->pdl_skip_once ? 1 : 0;
    h->pdl_skip_once = false;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

static moss_enc_status fail(moss_enc *h, moss_enc_status s, const std::string &msg)
{
    if (h) h->last_error = msg;
    return s;
}

#define CUDA_TRY(h, call)                                                                       \
    do {                                                                                        \
        cudaError_t e_ = (call);                                                                \
        if (e_ != cudaSuccess)                                                                  \
            return fail(h, MOSS_ENC_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
    } while (0)

typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                      const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                      const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled_t encode_fn()
{
    static PFN_encodeTiled_t fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled_t>(p);
    }
    return fn;
}

// 2-D bf16 tensor map: rows of `inner` elements, `row_bytes` apart; box of
// box_inner x box_rows with 128-byte swizzle (box_inner = 64).
static bool tmap_2d(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                    uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B)
{
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output map of the pair GEMM's TMA epilogue: [M][ldo] of bf16 (boxes of
// 64 columns x 32 rows) or fp32 (32 x 32), 128-byte swizzle to match the
// epilogue's staging layout.  Other epilogues get a copy of `fallback`
// (never read).
template <int BN, int EPI>
static bool tmap_out(CUtensorMap *m, const GemmArgs &a, const CUtensorMap &fallback)
{
    const bool f32 = EPI == EPI_RESID_F32 || EPI == EPI_F32;
    const bool tma = (BN % 64 == 0 && (f32 || EPI == EPI_BF16 || EPI == EPI_GELU_BF16)) || (BN % 64 == 32 && f32);
    if (!tma) {
        *m = fallback;
        return true;
    }
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return false;
    const uint64_t esz = f32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)a.ldo, (cuuint64_t)a.M};
    cuuint64_t strides[1] = {(cuuint64_t)a.ldo * esz};
    cuuint32_t box[2] = {f32 ? 32u : 64u, 32u};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.out, dims,
                    strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output bytes per element for the epilogue kinds (for the byte count).
static double epi_out_bytes(int epi)
{
    return epi == EPI_RESID_F32 ? 8.0 : (epi == EPI_F32 || epi == EPI_CONVOUT_F32) ? 4.0 : epi == EPI_SWIGLU_BF16 ? 1.0 : 2.0;
}

// k_alg: the contraction length the method needs (padding excluded).
template <int BN, int EPI>
static moss_enc_status gemm(moss_enc *h, const char *name, const bf16 *A, int64_t M, int K, const bf16 *B, int N,
                            GemmArgs a, int k_alg = 0)
{
    if (M <= 0) return MOSS_ENC_OK;
    if (K % 64 != 0 || N % BN != 0 || M > INT32_MAX)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "gemm shape not supported");
    CUtensorMap ta, tb;
    if (!tmap_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, 128) ||
        !tmap_2d(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, 64, BN))
        return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    a.M = (int)M;
    a.N = N;
    a.K = K;
    a.m_tiles = (int)((M + 127) / 128);
    a.n_tiles = N / BN;
    a.err = h->err;
    const int tiles = a.m_tiles * a.n_tiles;
    const int grid = std::min(tiles, h->num_sms);
    const double ka = k_alg > 0 ? k_alg : K;
    Launch L(h, name, 2.0 * M * N * ka, 2.0 * M * ka + 2.0 * N * ka + epi_out_bytes(EPI) * M * N);
    gemm_tc_kernel<BN, EPI><<<grid, GemmCfg<BN>::THREADS, GemmCfg<BN>::SMEM, h->stream>>>(ta, tb, a);
    CUDA_TRY(h, cudaGetLastError());
    return MOSS_ENC_OK;
}

// The same on CTA pairs (256-row tiles, cluster of 2).  ksub: 64-wide k
// sub-blocks per pipeline stage (2 when K allows it and the stages still fit
// at least three deep, i.e. BN <= 256; callers may ask for 1 or 2).
template <int BN, int EPI>
static moss_enc_status gemm2(moss_enc *h, const char *name, const bf16 *A, int64_t M, int K, const bf16 *B, int N,
                             GemmArgs a, int k_alg = 0, int ksub = BN <= 256 ? 2 : 1)
{
    if (M <= 0) return MOSS_ENC_OK;
    if (K % 64 != 0 || N % BN != 0 || M > INT32_MAX)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "gemm shape not supported");
    CUtensorMap ta, tb;
    if (!tmap_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, 128) ||
        !tmap_2d(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, 64, Gemm2Cfg<BN>::NS / 2))
        return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    a.M = (int)M;
    a.N = N;
    a.K = K;
    a.m_tiles = (int)((M + 255) / 256);
    a.n_tiles = N / BN;
    a.err = h->err;
    CUtensorMap tc;
    if (!tmap_out<BN, EPI>(&tc, a, tb)) return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (output)");
    const int tiles = a.m_tiles * a.n_tiles;
    const int grid = 2 * std::min(tiles, h->num_sms / 2);
    const double ka = k_alg > 0 ? k_alg : K;
    Launch L(h, name, 2.0 * M * N * ka, 2.0 * M * ka + 2.0 * N * ka + epi_out_bytes(EPI) * M * N);
    // 320-wide tiles of a launch with no more tiles than SM pairs: two k
    // sub-blocks per stage, three stages, output staged in the idle ring
    constexpr bool ring_ok = BN == 320 && (EPI == EPI_BF16 || EPI == EPI_GELU_BF16 || EPI == EPI_RESID_F32 || EPI == EPI_F32);
    if (ring_ok && tiles <= h->num_sms / 2 && K % 128 == 0)
        CUDA_TRY(h, launch_k(h, gemm_tc2_kernel<BN, EPI, A_PLAIN, 2, 0, 0, ring_ok ? 1 : 0>, dim3(grid),
                             dim3(Gemm2Cfg<BN, 2, 0, 1>::THREADS), Gemm2Cfg<BN, 2, 0, 1>::SMEM, ta, tb, tc, tb, a));
    else if (ksub == 2 && K % 128 == 0)
        CUDA_TRY(h, launch_k(h, gemm_tc2_kernel<BN, EPI, A_PLAIN, 2>, dim3(grid), dim3(Gemm2Cfg<BN, 2>::THREADS),
                             Gemm2Cfg<BN, 2>::SMEM, ta, tb, tc, tb, a));
    else
        CUDA_TRY(h, launch_k(h, gemm_tc2_kernel<BN, EPI, A_PLAIN, 1>, dim3(grid), dim3(Gemm2Cfg<BN, 1>::THREADS),
                             Gemm2Cfg<BN, 1>::SMEM, ta, tb, tc, tb, a));
    return MOSS_ENC_OK;
}

// The pair GEMM with a 4-bit B: the codes and scales stream in by TMA and
// converter warps expand them to bf16 in shared memory for the MMA.
template <int BN, int EPI>
static moss_enc_status gemm2q(moss_enc *h, const char *name, const bf16 *A, int64_t M, int K, const QW &B, int N,
                              GemmArgs a, int k_alg = 0)
{
    using C = Gemm2Cfg<BN, 1, 1>;
    if (M <= 0) return MOSS_ENC_OK;
    if (K % 64 != 0 || N % BN != 0 || M > INT32_MAX || B.kq % 128 != 0 || K % B.kq != 0)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "gemm shape not supported");
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return fail(h, MOSS_ENC_ERR_CUDA, "no tensor-map encoder");
    CUtensorMap ta, tq, ts;
    if (!tmap_2d(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, 128))
        return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    {
        // codes: [N][kq / 2] bytes, boxes of 32 bytes (64 k) x NS/2 rows
        cuuint64_t dims[2] = {(cuuint64_t)B.kq / 2, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)B.kq / 2};
        cuuint32_t box[2] = {32, (cuuint32_t)(C::NS / 2)};
        cuuint32_t es[2] = {1, 1};
        if (fn(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(B.codes), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (codes)");
    }
    {
        // scales: [kq / 128][N] fp32, boxes of NS/2 rows x 1 group
        cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)B.kq / 128};
        cuuint64_t strides[1] = {(cuuint64_t)N * 4};
        cuuint32_t box[2] = {(cuuint32_t)(C::NS / 2), 1};
        cuuint32_t es[2] = {1, 1};
        if (fn(&ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(B.scales), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (scales)");
    }
    a.M = (int)M;
    a.N = N;
    a.K = K;
    a.m_tiles = (int)((M + 255) / 256);
    a.n_tiles = N / BN;
    a.err = h->err;
    a.kq_blocks = B.kq / 64;
    CUtensorMap tc;
    if (!tmap_out<BN, EPI>(&tc, a, tq)) return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (output)");
    const int tiles = a.m_tiles * a.n_tiles;
    const int grid = 2 * std::min(tiles, h->num_sms / 2);
    const double ka = k_alg > 0 ? k_alg : K;
    Launch L(h, name, 2.0 * M * N * ka, 2.0 * M * ka + 0.5 * N * (double)B.kq + 4.0 * N * (B.kq / 128) +
                                            epi_out_bytes(EPI) * M * N);
    CUDA_TRY(h, launch_k(h, gemm_tc2_kernel<BN, EPI, A_PLAIN, 1, 1>, dim3(grid), dim3(C::THREADS), C::SMEM, ta, tq, tc,
                         ts, a));
    return MOSS_ENC_OK;
}

// The pair GEMM on e4m3 operands: A8 [M][K] and B8 [N][K] bytes, row scales
// a.row_scale [M] and column scales a.col_scale [N] applied in the epilogue
// (bf16 outputs).  Two 128-wide k rows per stage.
template <int BN, int EPI>
static moss_enc_status gemm2f8(moss_enc *h, const char *name, const uint8_t *A8, int64_t M, int K, const uint8_t *B8,
                               int N, GemmArgs a)
{
    using C = Gemm2Cfg<BN, 2>;
    if (M <= 0) return MOSS_ENC_OK;
    if (K % 256 != 0 || N % BN != 0 || M > INT32_MAX || !a.row_scale || !a.col_scale)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "gemm shape not supported");
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return fail(h, MOSS_ENC_ERR_CUDA, "no tensor-map encoder");
    CUtensorMap ta, tb;
    auto map8 = [&](CUtensorMap *m, const uint8_t *p, uint64_t rows, uint32_t box_rows) {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
        cuuint64_t strides[1] = {(cuuint64_t)K};
        cuuint32_t box[2] = {128, box_rows};
        cuuint32_t es[2] = {1, 1};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(p), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    if (!map8(&ta, A8, (uint64_t)M, 128) || !map8(&tb, B8, (uint64_t)N, C::NS / 2))
        return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (e4m3)");
    a.M = (int)M;
    a.N = N;
    a.K = K;
    a.m_tiles = (int)((M + 255) / 256);
    a.n_tiles = N / BN;
    a.err = h->err;
    CUtensorMap tc;
    if (!tmap_out<BN, EPI>(&tc, a, tb)) return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (output)");
    const int tiles = a.m_tiles * a.n_tiles;
    const int grid = 2 * std::min(tiles, h->num_sms / 2);
    Launch L(h, name, 2.0 * M * N * K, 1.0 * M * K + 1.0 * N * K + epi_out_bytes(EPI) * M * N);
    CUDA_TRY(h, launch_k(h, gemm_tc2_kernel<BN, EPI, A_PLAIN, 2, 0, 1>, dim3(grid), dim3(C::THREADS), C::SMEM, ta, tb, tc,
                         tb, a));
    return MOSS_ENC_OK;
}

// The NVFP4 GEMM (fp4.cuh): A4 [M][K/2] and B4 [N][K/2] E2M1 bytes, their
// block-scale atoms a.sfa and a.sfb, row factors a.row_scale [M] (g of each
// activation row) and column factors a.col_scale [N] (the weight's g);
// bf16 outputs.  128 x 128 tiles, 256 k per stage.
template <int EPI>
static moss_enc_status gemm_nvf4(moss_enc *h, const char *name, const uint8_t *A4, int64_t M, int K, const uint8_t *B4,
                                 int N, GemmArgs a)
{
    using C = Fp4Cfg<128>;
    if (M <= 0) return MOSS_ENC_OK;
    if (K % 256 != 0 || N % 128 != 0 || M > INT32_MAX || !a.row_scale || !a.col_scale || !a.sfa || !a.sfb)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "gemm shape not supported");
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return fail(h, MOSS_ENC_ERR_CUDA, "no tensor-map encoder");
    CUtensorMap ta, tb;
    auto map4 = [&](CUtensorMap *m, const uint8_t *p, uint64_t rows) {
        cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)rows};
        cuuint64_t strides[1] = {(cuuint64_t)K / 2};
        cuuint32_t box[2] = {128, 128};
        cuuint32_t es[2] = {1, 1};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(p), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    if (!map4(&ta, A4, (uint64_t)M) || !map4(&tb, B4, (uint64_t)N))
        return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (fp4)");
    a.M = (int)M;
    a.N = N;
    a.K = K;
    a.m_tiles = (int)((M + 127) / 128);
    a.n_tiles = N / 128;
    a.err = h->err;
    CUtensorMap tc;
    if (!tmap_out<128, EPI>(&tc, a, tb)) return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (output)");
    const int tiles = a.m_tiles * a.n_tiles;
    const int grid = std::min(tiles, h->num_sms);
    Launch L(h, name, 2.0 * M * N * K, 0.5 * M * K + 0.5 * N * K + (M + N) * K / 16.0 + epi_out_bytes(EPI) * M * N);
    CUDA_TRY(h, launch_k(h, gemm_nvf4_kernel<128, EPI>, dim3(grid), dim3(C::THREADS), C::SMEM, ta, tb, tc, a));
    return MOSS_ENC_OK;
}

template <int BN, int EPI>
static cudaError_t gemm2f8_attr()
{
    return cudaFuncSetAttribute(gemm_tc2_kernel<BN, EPI, A_PLAIN, 2, 0, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Gemm2Cfg<BN, 2>::SMEM);
}

template <int BN, int EPI>
static cudaError_t gemm2q_attr()
{
    return cudaFuncSetAttribute(gemm_tc2_kernel<BN, EPI, A_PLAIN, 1, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Gemm2Cfg<BN, 1, 1>::SMEM);
}

template <int BN, int EPI>
static cudaError_t gemm2_attr()
{
    cudaError_t e = cudaFuncSetAttribute(gemm_tc2_kernel<BN, EPI, A_PLAIN, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Gemm2Cfg<BN, 1>::SMEM);
    if (e != cudaSuccess) return e;
    constexpr bool ring_ok = BN == 320 && (EPI == EPI_BF16 || EPI == EPI_GELU_BF16 || EPI == EPI_RESID_F32 || EPI == EPI_F32);
    if (ring_ok) {
        e = cudaFuncSetAttribute(gemm_tc2_kernel<BN, EPI, A_PLAIN, 2, 0, 0, ring_ok ? 1 : 0>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Gemm2Cfg<BN, 2, 0, 1>::SMEM);
        if (e != cudaSuccess) return e;
    }
    return cudaFuncSetAttribute(gemm_tc2_kernel<BN, EPI, A_PLAIN, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Gemm2Cfg<BN, 2>::SMEM);
}

#define TRY(x)                                  \
    do {                                        \
        moss_enc_status s_ = (x);               \
        if (s_ != MOSS_ENC_OK) return s_;       \
    } while (0)

// 4-D bf16 map over NHWC [chunks][Ti][Fi][480] whose box holds the inputs of
// one 128-row output tile of a 3x3 stride-2 conv: 64 channels x Fo
// frequencies x tile_t time steps, both spatial axes traversed with stride 2.
static bool tmap_conv(CUtensorMap *m, const void *ptr, int chunks, int Ti, int Fi, int tile_t)
{
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return false;
    const int Fo = (Fi + 1) / 2;
    cuuint64_t dims[4] = {480, (cuuint64_t)Fi, (cuuint64_t)Ti, (cuuint64_t)chunks};
    cuuint64_t strides[3] = {480 * 2, (cuuint64_t)Fi * 480 * 2, (cuuint64_t)Ti * Fi * 480 * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)(2 * Fo), (cuuint32_t)(2 * tile_t), 1};
    cuuint32_t es[4] = {1, 2, 2, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// conv2/conv3 as an implicit GEMM on CTA pairs: out [chunk][To][Fo][480] =
// GELU(conv(in) + b) for the 128-row tiles listed in d_tiles (n_items of
// them, padded with -1 to an even count; CTA r of pair p takes item 2p + r).
static moss_enc_status gemm_conv(moss_enc *h, const char *name, const bf16 *in, int chunks, int Ti, int Fi,
                                 const int *d_tiles, int n_items, const bf16 *W, const float *bias, bf16 *out)
{
    if (n_items <= 0) return MOSS_ENC_OK;
    const int Fo = (Fi + 1) / 2, To = (Ti + 1) / 2, tile_t = 128 / Fo;
    CUtensorMap ta, tb;
    if (!tmap_conv(&ta, in, chunks, Ti, Fi, tile_t) ||
        !tmap_2d(&tb, W, (uint64_t)CONV_K, (uint64_t)CST, (uint64_t)CONV_K * 2, 64, CONV_BN / 2))
        return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (conv)");
    GemmArgs a{};
    a.M = n_items * 128;
    a.N = CST;
    a.K = CONV_K;
    a.m_tiles = (n_items + 1) / 2;
    a.n_tiles = CST / CONV_BN;
    a.err = h->err;
    a.bias = bias;
    a.out = out;
    a.ldo = CST;
    a.tile_list = d_tiles;
    a.rows_per_chunk = To * Fo;
    a.tile_t = tile_t;
    const int grid = 2 * std::min(a.m_tiles * a.n_tiles, h->num_sms / 2);
    Launch L(h, name, 2.0 * 128.0 * n_items * CST * (9.0 * CST), 2.0 * 128.0 * n_items * (9.0 * CST) * 0.25 + 2.0 * 128.0 * n_items * CST);
    CUDA_TRY(h, launch_k(h, gemm_tc2_kernel<CONV_BN, EPI_GELU_BF16, A_CONV_S2, 2>, dim3(grid),
                         dim3(Gemm2Cfg<CONV_BN, 2>::THREADS), Gemm2Cfg<CONV_BN, 2>::SMEM, ta, tb, tb, tb, a));
    return MOSS_ENC_OK;
}

template <int BN, int EPI>
static cudaError_t gemm_attr()
{
    return cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)GemmCfg<BN>::SMEM);
}

static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// ------------------------------------------------------ host-side constants

// Slaney mel scale (linear below 1 kHz at 200/3 Hz per mel, logarithmic above
// with a step of ln(6.4)/27 per mel).
static double slaney_mel(double hz)
{
    return hz < 1000.0 ? hz * 3.0 / 200.0 : 15.0 + std::log(hz / 1000.0) * 27.0 / std::log(6.4);
}

static double slaney_hz(double mel)
{
    return mel < 15.0 ? mel * 200.0 / 3.0 : 1000.0 * std::exp((mel - 15.0) * std::log(6.4) / 27.0);
}

// Twiddles, periodic Hann and the banded 128 x 201 Slaney filterbank
// (triangles between mel-spaced edges over 0..8 kHz, area-normalised).
static bool build_mel_tables(MelTables *t)
{
    for (int k = 0; k < 400; k++) {
        const double a = -2.0 * M_PI * k / 400.0;
        t->tw400[k] = make_float2((float)std::cos(a), (float)std::sin(a));
        t->hann[k] = (float)(0.5 - 0.5 * std::cos(2.0 * M_PI * k / 400.0));
    }
    double edge[130];
    const double top = slaney_mel(8000.0);
    for (int i = 0; i < 130; i++) edge[i] = slaney_hz(top * i / 129.0);
    for (int m = 0; m < 128; m++) {
        double w[201];
        int lo = -1, hi = -1;
        for (int k = 0; k <= 200; k++) {
            const double f = 40.0 * k;
            const double rise = (f - edge[m]) / (edge[m + 1] - edge[m]);
            const double fall = (edge[m + 2] - f) / (edge[m + 2] - edge[m + 1]);
            double v = std::min(rise, fall);
            v = v > 0.0 ? v * 2.0 / (edge[m + 2] - edge[m]) : 0.0;
            w[k] = v;
            if (v > 0.0) {
                if (lo < 0) lo = k;
                hi = k;
            }
        }
        if (lo < 0) lo = hi = 0;
        if (hi - lo + 1 > MEL_BAND) return false;
        t->band_lo[m] = lo;
        t->band_n[m] = hi - lo + 1;
        for (int b = 0; b < MEL_BAND; b++) t->band_w[m][b] = (lo + b <= 200) ? (float)w[lo + b] : 0.0f;
    }
    return true;
}

// The persistent log-mel kernel's tables in its shared-memory layout: the
// twiddles w^(n1 k2) at [k2][n1], the window, the filterbank as 32 groups of
// 4 filters (first bins, bin pairs to visit, the weights of each bin pair as
// float4 over the group's filters), and the groups of each warp, balanced by
// their work in the kernel (a fixed part for the shuffles, logs and stores,
// plus the bin pairs).
static bool build_mel4_tab(const MelTables &t, Mel4Tab *o)
{
    std::memset(o, 0, sizeof(Mel4Tab));
    for (int k2 = 0; k2 < 20; k2++)
        for (int n1 = 0; n1 < 21; n1++) o->tw[k2][n1] = n1 < 20 ? t.tw400[(n1 * k2) % 400] : make_float2(0.0f, 0.0f);
    for (int i = 0; i < 400; i++) o->hann[i] = t.hann[i];
    int cost[MEL4_GROUPS], total = 0, woff = 0;
    for (int g = 0; g < MEL4_GROUPS; g++) {
        Mel4Group &G = o->grp[g];
        int nmax = 0;
        for (int j = 0; j < 4; j++) {
            G.lo[j] = t.band_lo[4 * g + j];
            nmax = std::max(nmax, t.band_n[4 * g + j]);
        }
        G.nit = (nmax + 1) / 2;
        G.woff = woff;
        for (int it = 0; it < G.nit; it++)
            for (int h = 0; h < 2; h++) {
                float w[4];
                for (int j = 0; j < 4; j++) {
                    const int b = 2 * it + h, m = 4 * g + j;
                    w[j] = b < t.band_n[m] ? t.band_w[m][b] : 0.0f;
                }
                o->w4[woff + 2 * it + h] = make_float4(w[0], w[1], w[2], w[3]);
            }
        woff += 2 * G.nit;
        if (woff > MEL4_GROUPS * MEL4_MAXIT * 2) return false;
        cost[g] = 40 + 10 * G.nit;
        total += cost[g];
    }
    int w = 0, run = 0;
    o->gpart[0] = 0;
    for (int g = 0; g < MEL4_GROUPS; g++) {
        run += cost[g];
        while (w + 1 < MEL4_WARPS && run * MEL4_WARPS >= total * (w + 1)) o->gpart[++w] = g + 1;
    }
    while (w + 1 <= MEL4_WARPS) o->gpart[++w] = MEL4_GROUPS;
    return true;
}

// ----------------------------------------------------------------- sizes

extern "C" int64_t moss_enc_weight_count(int n_layers)
{
    if (n_layers < 0) return -1;
    int64_t n = (int64_t)CST * 9 + CST + 2 * ((int64_t)CST * CST * 9 + CST) + (int64_t)D * CST * 16;
    const int64_t per_layer = 4 * (int64_t)D + 4 * ((int64_t)D * D + D) + ((int64_t)DFF * D + DFF) +
                              ((int64_t)D * DFF + D);
    n += per_layer * n_layers;
    n += 2 * (int64_t)D + ((int64_t)D * D + D) + ((int64_t)DOUT * D + DOUT);
    n += 2 * ((int64_t)DADP * DOUT + DADP) + ((int64_t)DOUT * DADP + DOUT);
    return n;
}

extern "C" int64_t moss_enc_num_frames(int64_t n_samples) { return n_samples <= 0 ? 0 : n_samples / HOP; }

static int64_t chunk_tokens(int64_t frames) { return (frames + 7) / 8; }

static bool plan_clip(int64_t n, int64_t begin, int64_t end, ClipPlan *p)
{
    if (n < 0 || begin < 0 || end > n || begin > end) return false;
    if (begin % CHUNK_SAMPLES != 0) return false;
    if (end != n && end % CHUNK_SAMPLES != 0) return false;
    p->n = n;
    p->F = moss_enc_num_frames(n);
    p->f_begin = begin / HOP;
    p->f_end = end == n ? p->F : end / HOP;
    if (p->f_begin > p->f_end) p->f_begin = p->f_end;
    p->c_first = p->f_begin / CHUNK_FRAMES;
    p->c_last = (p->f_end + CHUNK_FRAMES - 1) / CHUNK_FRAMES;
    if (p->f_end <= p->f_begin) p->c_last = p->c_first;
    p->ntok = 0;
    for (int64_t c = p->c_first; c < p->c_last; c++)
        p->ntok += chunk_tokens(std::min<int64_t>(CHUNK_FRAMES, p->F - c * CHUNK_FRAMES));
    return true;
}

extern "C" int64_t moss_enc_num_tokens(int64_t n_samples)
{
    ClipPlan p;
    if (!plan_clip(n_samples < 0 ? 0 : n_samples, 0, n_samples < 0 ? 0 : n_samples, &p)) return -1;
    return p.ntok;
}

extern "C" int64_t moss_enc_range_tokens(int64_t n_samples, int64_t begin, int64_t end)
{
    ClipPlan p;
    if (!plan_clip(n_samples, begin, end, &p)) return -1;
    return p.ntok;
}

extern "C" const char *moss_enc_status_string(moss_enc_status s)
{
    switch (s) {
    case MOSS_ENC_OK: return "ok";
    case MOSS_ENC_ERR_INVALID_ARG: return "invalid argument";
    case MOSS_ENC_ERR_CAPACITY: return "request exceeds capacity";
    case MOSS_ENC_ERR_OOM: return "out of device memory";
    case MOSS_ENC_ERR_CUDA: return "CUDA error";
    case MOSS_ENC_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

extern "C" const char *moss_enc_last_error(const moss_enc *h) { return h ? h->last_error.c_str() : ""; }

// ------------------------------------------------------------ create/destroy

// Table layout inside the per-call staging area.
struct TabLayout {
    size_t clips_main, clips_max, chunks, chunk_tok, logmax_src, tiles2, tiles3, total;
};

static TabLayout tab_layout(int64_t max_clips, int64_t max_chunks)
{
    TabLayout t;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t r = o;
        o += (bytes + 255) & ~size_t(255);
        return r;
    };
    t.clips_main = take(sizeof(MelClip) * max_clips);
    t.clips_max = take(sizeof(MelClip) * max_clips);
    t.chunks = take(sizeof(StemChunk) * max_chunks);
    t.chunk_tok = take(sizeof(int2) * max_chunks);
    t.logmax_src = take(sizeof(float *) * max_clips);
    t.tiles2 = take(sizeof(int) * (max_chunks * C2_TILES + max_chunks));
    t.tiles3 = take(sizeof(int) * (max_chunks * C3_TILES + max_chunks));
    t.total = o;
    return t;
}

extern "C" void moss_enc_destroy(moss_enc *h)
{
    if (!h) return;
    cudaSetDevice(h->device);
    if (h->stream) cudaStreamSynchronize(h->stream);
    else cudaDeviceSynchronize();
    if (h->wmem) cudaFree(h->wmem);
    if (h->qmem) cudaFree(h->qmem);
    if (h->tap_wmem) cudaFree(h->tap_wmem);
    if (h->ws) cudaFree(h->ws);
    if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
    if (h->d_tab) cudaFree(h->d_tab);
    if (h->d_tab_graph) cudaFree(h->d_tab_graph);
    if (h->h_tab_ring) cudaFreeHost(h->h_tab_ring);
    for (cudaEvent_t e : h->tab_event)
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
    delete h;
}

// Packed layout of one head + adapter set (ln_post, proj1, proj2, gate/up,
// down).  proj1 and proj2 are stored twice along K ([W | W]) for the split
// [hi | lo] operands; gate and up are interleaved in blocks of 32 output
// rows: g[0:32], u[0:32], g[32:64], ...
struct HeadOff {
    size_t lnp, p1, bp1, p2, bp2, gu, bgu, wd, bd;
};

// The small tensors are taken with `small`, the four weight matrices with
// `big` (the encoder's own set keeps them in the part a 4-bit handle
// replaces by codes).
template <class TakeS, class TakeB>
static HeadOff head_take(TakeS &small, TakeB &big)
{
    HeadOff o;
    o.lnp = small(4 * 2 * D);
    o.bp1 = small(4 * D);
    o.bp2 = small(4 * DOUT);
    o.bgu = small(4 * 2 * DADP);
    o.bd = small(4 * DOUT);
    o.p1 = big(2 * (size_t)D * 2 * D);
    o.p2 = big(2 * (size_t)DOUT * 2 * D);
    o.gu = big(2 * (size_t)2 * DADP * DOUT);
    o.wd = big(2 * (size_t)DOUT * DADP);
    return o;
}

// bf16 elements of one head + adapter set in the blob order: ln_post.g,
// ln_post.b, proj1.w, proj1.b, proj2.w, proj2.b, gate.w, gate.b, up.w, up.b,
// down.w, down.b.
static int64_t head_count()
{
    return 2 * (int64_t)D + (int64_t)D * D + D + (int64_t)DOUT * D + DOUT + 2 * ((int64_t)DADP * DOUT + DADP) +
           (int64_t)DOUT * DADP + DOUT;
}

// Repacks one set from the blob order at p into pk; returns the end of it.
static const uint16_t *head_pack(const HeadOff &o, uint8_t *pk, const uint16_t *p)
{
    auto F32 = [&](size_t off) { return reinterpret_cast<float *>(pk + off); };
    auto U16 = [&](size_t off) { return reinterpret_cast<uint16_t *>(pk + off); };
    auto copy_twice = [&](uint16_t *dst, const uint16_t *src_rows, int rows, int k) {
        for (int r = 0; r < rows; r++) {
            std::memcpy(dst + (size_t)r * 2 * k, src_rows + (size_t)r * k, 2 * (size_t)k);
            std::memcpy(dst + (size_t)r * 2 * k + k, src_rows + (size_t)r * k, 2 * (size_t)k);
        }
    };
    for (int i = 0; i < 2 * D; i++) F32(o.lnp)[i] = bf16_bits_to_float(p[i]);
    p += 2 * D;
    copy_twice(U16(o.p1), p, D, D);
    p += (size_t)D * D;
    for (int i = 0; i < D; i++) F32(o.bp1)[i] = bf16_bits_to_float(p[i]);
    p += D;
    copy_twice(U16(o.p2), p, DOUT, D);
    p += (size_t)DOUT * D;
    for (int i = 0; i < DOUT; i++) F32(o.bp2)[i] = bf16_bits_to_float(p[i]);
    p += DOUT;
    const uint16_t *gw = p;
    const uint16_t *gb = gw + (size_t)DADP * DOUT;
    const uint16_t *uw = gb + DADP;
    const uint16_t *ub = uw + (size_t)DADP * DOUT;
    for (int j = 0; j < DADP / 32; j++)
        for (int r = 0; r < 32; r++) {
            std::memcpy(U16(o.gu) + ((size_t)(64 * j + r)) * DOUT, gw + (size_t)(32 * j + r) * DOUT, 2 * (size_t)DOUT);
            std::memcpy(U16(o.gu) + ((size_t)(64 * j + 32 + r)) * DOUT, uw + (size_t)(32 * j + r) * DOUT, 2 * (size_t)DOUT);
            F32(o.bgu)[64 * j + r] = bf16_bits_to_float(gb[32 * j + r]);
            F32(o.bgu)[64 * j + 32 + r] = bf16_bits_to_float(ub[32 * j + r]);
        }
    p = ub + DADP;
    std::memcpy(U16(o.wd), p, 2 * (size_t)DOUT * DADP);
    p += (size_t)DOUT * DADP;
    for (int i = 0; i < DOUT; i++) F32(o.bd)[i] = bf16_bits_to_float(p[i]);
    return p + DOUT;
}

static HeadDev head_bind(const HeadOff &o, uint8_t *W)
{
    HeadDev d;
    d.lnp_g = (float *)(W + o.lnp);
    d.lnp_b = d.lnp_g + D;
    d.wp1 = (bf16 *)(W + o.p1);
    d.bp1 = (float *)(W + o.bp1);
    d.wp2 = (bf16 *)(W + o.p2);
    d.bp2 = (float *)(W + o.bp2);
    d.wgu = (bf16 *)(W + o.gu);
    d.bgu = (float *)(W + o.bgu);
    d.wd = (bf16 *)(W + o.wd);
    d.bd = (float *)(W + o.bd);
    return d;
}

static moss_enc_status set_kernel_attrs(moss_enc *h)
{
    CUDA_TRY(h, cudaFuncSetAttribute(gemm_tc2_kernel<CONV_BN, EPI_GELU_BF16, A_CONV_S2, 2>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Gemm2Cfg<CONV_BN, 2>::SMEM));
    CUDA_TRY(h, (gemm2_attr<256, EPI_BF16>()));
    CUDA_TRY(h, (gemm2_attr<256, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm2_attr<320, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm2_attr<128, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm2_attr<160, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm2_attr<128, EPI_F32>()));
    CUDA_TRY(h, (gemm2f8_attr<128, EPI_BF16>()));
    CUDA_TRY(h, cudaFuncSetAttribute(gemm_nvf4_kernel<128, EPI_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)Fp4Cfg<128>::SMEM));
    CUDA_TRY(h, cudaFuncSetAttribute(gemm_nvf4_kernel<128, EPI_GELU_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)Fp4Cfg<128>::SMEM));
    CUDA_TRY(h, (gemm2f8_attr<256, EPI_BF16>()));
    CUDA_TRY(h, (gemm2f8_attr<128, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm2f8_attr<256, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm2q_attr<128, EPI_BF16>()));
    CUDA_TRY(h, (gemm2q_attr<256, EPI_BF16>()));
    CUDA_TRY(h, (gemm2q_attr<128, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm2q_attr<160, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm2q_attr<320, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm2q_attr<256, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm2q_attr<320, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm2q_attr<256, EPI_F32>()));
    CUDA_TRY(h, (gemm2q_attr<256, EPI_SWIGLU_BF16>()));
    CUDA_TRY(h, (gemm2q_attr<128, EPI_F32>()));
    CUDA_TRY(h, (gemm2_attr<128, EPI_BF16>()));
    CUDA_TRY(h, (gemm2_attr<320, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm2_attr<256, EPI_SWIGLU_BF16>()));
    CUDA_TRY(h, (gemm2_attr<256, EPI_F32>()));
    CUDA_TRY(h, (gemm2_attr<256, EPI_BF16>()));
    CUDA_TRY(h, (gemm2_attr<320, EPI_CONVOUT_F32>()));
    CUDA_TRY(h, (gemm_attr<160, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm_attr<160, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm_attr<256, EPI_BF16>()));
    CUDA_TRY(h, (gemm_attr<128, EPI_CONVOUT_F32>()));
    CUDA_TRY(h, (gemm_attr<256, EPI_BF16>()));
    CUDA_TRY(h, (gemm_attr<256, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm_attr<128, EPI_RESID_F32>()));
    CUDA_TRY(h, (gemm_attr<128, EPI_GELU_BF16>()));
    CUDA_TRY(h, (gemm_attr<256, EPI_F32>()));
    CUDA_TRY(h, (gemm_attr<256, EPI_SWIGLU_BF16>()));
    CUDA_TRY(h, (gemm_attr<128, EPI_F32>()));
    CUDA_TRY(h, (gemm_attr<128, EPI_BF16>()));
    CUDA_TRY(h, cudaFuncSetAttribute(window_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ATTN_TC_SMEM));
    CUDA_TRY(h, cudaFuncSetAttribute(conv1_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C1_SMEM));
    CUDA_TRY(h, cudaFuncSetAttribute(logmel4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Mel4Smem)));
    CUDA_TRY(h, cudaFuncSetAttribute(logmel4_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
    return MOSS_ENC_OK;
}

// e4m3 quantisation of a bf16 matrix [n][k] in place, per row: s = fp32(max
// |w|) / 448, codes e4m3(w / s) (round to nearest even, saturating) as bytes
// [n][k] from the matrix's start, then the scales [n] at f8_scale_off.  A
// zero row has scale 0 and zero codes.
static size_t f8_scale_off(int n, int k) { return ((size_t)n * k + 255) & ~size_t(255); }

static void quantise_e4m3_rows(uint8_t *mat, int n, int k)
{
    std::vector<uint8_t> codes((size_t)n * k);
    std::vector<float> sc(n);
    const uint16_t *w = reinterpret_cast<const uint16_t *>(mat);
    for (int r = 0; r < n; r++) {
        float amax = 0.0f;
        for (int i = 0; i < k; i++) amax = std::max(amax, std::fabs(bf16_bits_to_float(w[(size_t)r * k + i])));
        const float s = amax / 448.0f;
        sc[r] = s;
        for (int i = 0; i < k; i++)
            codes[(size_t)r * k + i] =
                s > 0.0f ? (uint8_t)__nv_cvt_float_to_fp8(bf16_bits_to_float(w[(size_t)r * k + i]) / s, __NV_SATFINITE,
                                                          __NV_E4M3)
                         : 0;
    }
    std::memcpy(mat, codes.data(), codes.size());
    std::memcpy(mat + f8_scale_off(n, k), sc.data(), sizeof(float) * n);
}

// NVFP4 quantisation of a bf16 matrix [n][k] in place (n a multiple of 128,
// k of 64), in `parts` equal row ranges with a g each (the q, k and v
// weights of the fused QKV matrix keep their own): g = fp32(amax) / 2688,
// s_b = e4m3(fp32(amax_b) / (g * 6)) per 16 k, code = e2m1(w / (s_b * g))
// (0 when s_b = 0; fp32 arithmetic, ties to even).  Written over the
// matrix: codes [n][k/2] (even k in the low nibble) from its start, the
// scale atoms [n/128][k/64][512] at nvf4_sf_off, g per row at nvf4_g_off.
static size_t nvf4_sf_off(int n, int k) { return ((size_t)n * k / 2 + 255) & ~size_t(255); }
static size_t nvf4_g_off(int n, int k) { return (nvf4_sf_off(n, k) + (size_t)n * k / 16 + 255) & ~size_t(255); }

// E2M1 code (sign bit 3, magnitude index 0..7 of 0, .5, 1, 1.5, 2, 3, 4, 6)
// of the value nearest to x; a tie goes to the even index; |x| > 6 -> 6.
static uint8_t host_e2m1(float x)
{
    static const float mid[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
    const float a = std::fabs(x);
    int i = 0;
    while (i < 7 && (a > mid[i] || (a == mid[i] && (i & 1)))) i++;
    return (uint8_t)(i | (std::signbit(x) ? 8 : 0));
}

static void quantise_nvfp4_to(const uint16_t *w, int n, int k, int parts, uint8_t *codes, uint8_t *atoms, float *gr)
{
    const int rows = n / parts;
    for (int p = 0; p < parts; p++) {
        float amax = 0.0f;
        for (size_t i = (size_t)p * rows * k; i < (size_t)(p + 1) * rows * k; i++)
            amax = std::max(amax, std::fabs(bf16_bits_to_float(w[i])));
        const float g = amax / 2688.0f;
        for (int r = p * rows; r < (p + 1) * rows; r++) {
            gr[r] = g;
            for (int b = 0; b < k / 16; b++) {
                float bmax = 0.0f;
                for (int i = 0; i < 16; i++) bmax = std::max(bmax, std::fabs(bf16_bits_to_float(w[(size_t)r * k + 16 * b + i])));
                const __nv_fp8_storage_t sc = g > 0.0f ? __nv_cvt_float_to_fp8(bmax / (g * 6.0f), __NV_SATFINITE, __NV_E4M3)
                                                       : (__nv_fp8_storage_t)0;
                const float sb = __half2float(__half(__nv_cvt_fp8_to_halfraw(sc, __NV_E4M3)));
                const float sg = sb * g;
                atoms[((size_t)(r / 128) * (k / 64) + b / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + b % 4] = sc;
                for (int i = 0; i < 16; i += 2) {
                    const size_t e = (size_t)r * k + 16 * b + i;
                    const uint8_t c0 = sb > 0.0f ? host_e2m1(bf16_bits_to_float(w[e]) / sg) : 0;
                    const uint8_t c1 = sb > 0.0f ? host_e2m1(bf16_bits_to_float(w[e + 1]) / sg) : 0;
                    codes[e / 2] = (uint8_t)(c0 | (c1 << 4));
                }
            }
        }
    }
}

static void quantise_nvfp4(uint8_t *mat, int n, int k, int parts)
{
    std::vector<uint8_t> codes((size_t)n * k / 2), atoms((size_t)n * k / 16);
    std::vector<float> gr(n);
    quantise_nvfp4_to(reinterpret_cast<const uint16_t *>(mat), n, k, parts, codes.data(), atoms.data(), gr.data());
    std::memcpy(mat, codes.data(), codes.size());
    std::memcpy(mat + nvf4_sf_off(n, k), atoms.data(), atoms.size());
    std::memcpy(mat + nvf4_g_off(n, k), gr.data(), sizeof(float) * n);
}

// 4-bit round-to-nearest quantisation of one bf16 matrix [n][kq] (rows
// `stride` elements apart) in groups of 128 along k: s = fp32(max |w|) / 7,
// q = clamp(rint(w / s), -8, 7) (0 when s = 0), code q + 8.  Codes [n][kq/2]
// (even k in the low nibble), scales [kq/128][n].
static void quantise_rows(const uint16_t *w, int r0, int r1, int n, int kq, int stride, uint8_t *codes, float *scales)
{
    const int groups = kq / 128;
    for (int r = r0; r < r1; r++)
        for (int g = 0; g < groups; g++) {
            const uint16_t *x = w + (size_t)r * stride + (size_t)g * 128;
            float amax = 0.0f;
            for (int i = 0; i < 128; i++) amax = std::max(amax, std::fabs(bf16_bits_to_float(x[i])));
            const float s = amax / 7.0f;
            scales[(size_t)g * n + r] = s;
            uint8_t *c = codes + (size_t)r * (kq / 2) + (size_t)g * 64;
            for (int i = 0; i < 128; i += 2) {
                int u[2];
                for (int e = 0; e < 2; e++) {
                    float q = 0.0f;
                    if (s > 0.0f) q = std::min(7.0f, std::max(-8.0f, std::rint(bf16_bits_to_float(x[i + e]) / s)));
                    u[e] = (int)q + 8;
                }
                c[i / 2] = (uint8_t)(u[0] | (u[1] << 4));
            }
        }
}

template <class QS>
static void quantise_all(const uint8_t *pk, uint8_t *qk, const QS *qs, size_t nq)
{
    const unsigned nt = std::max(1u, std::min(32u, std::thread::hardware_concurrency()));
    std::vector<std::thread> pool;
    for (unsigned t = 0; t < nt; t++)
        pool.emplace_back([&, t]() {
            for (size_t i = 0; i < nq; i++) {
                const QS &q = qs[i];
                const int r0 = (int)((int64_t)q.n * t / nt), r1 = (int)((int64_t)q.n * (t + 1) / nt);
                quantise_rows(reinterpret_cast<const uint16_t *>(pk + q.bf_off), r0, r1, q.n, q.kq, q.stride, qk + q.q_off,
                              reinterpret_cast<float *>(qk + q.s_off));
            }
        });
    for (auto &th : pool) th.join();
}

extern "C" moss_enc_status moss_enc_create(const moss_enc_config *cfg, const void *weights, size_t bytes,
                                           int weights_on_device, void *stream, moss_enc **out)
{
    if (!out) return MOSS_ENC_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg || !weights || cfg->n_layers < 1 || cfg->n_layers > 32 || cfg->max_samples < 1 ||
        cfg->max_clips < 1 || (cfg->out_dtype != MOSS_ENC_OUT_F32 && cfg->out_dtype != MOSS_ENC_OUT_BF16) ||
        (cfg->weight_bits != 0 && cfg->weight_bits != 16 && cfg->weight_bits != 4) ||
        (cfg->fp8 != 0 && cfg->fp8 != 1) || (cfg->fp8 && cfg->weight_bits == 4) ||
        (cfg->nvfp4 != 0 && cfg->nvfp4 != 1) || (cfg->nvfp4 && (cfg->fp8 || cfg->weight_bits == 4)))
        return MOSS_ENC_ERR_INVALID_ARG;
    const int64_t count = moss_enc_weight_count(cfg->n_layers);
    if ((int64_t)bytes != count * 2) return MOSS_ENC_ERR_INVALID_ARG;

    moss_enc *h = new (std::nothrow) moss_enc();
    if (!h) return MOSS_ENC_ERR_OOM;
    h->cfg = *cfg;
    h->stream = (cudaStream_t)stream;
    moss_enc_status st = MOSS_ENC_OK;
    auto bail = [&](moss_enc_status s) {
        moss_enc_destroy(h);
        return s;
    };
    if (cudaGetDevice(&h->device) != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, h->device) != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);
    if (prop.major != 10) return bail(MOSS_ENC_ERR_CUDA);  // built for sm_100a only
    h->num_sms = prop.multiProcessorCount;
    if (const char *e = std::getenv("MOSS_ENC_PDL")) h->pdl = std::strcmp(e, "0") != 0;
    if (!encode_fn()) return bail(MOSS_ENC_ERR_CUDA);
    if ((st = set_kernel_attrs(h)) != MOSS_ENC_OK) return bail(st);

    // ---- host copy of the blob
    std::vector<uint16_t> host;
    const uint16_t *src = static_cast<const uint16_t *>(weights);
    if (weights_on_device) {
        host.resize(count);
        if (cudaMemcpy(host.data(), weights, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);
        src = host.data();
    }

    // ---- sizes of the packed weights: the small tensors first, then the
    // weight matrices of the linear layers (the part a 4-bit handle keeps as
    // codes and scales only)
    const int L = cfg->n_layers;
    size_t off = 0;
    auto take = [&](size_t b) {
        size_t r = off;
        off += (b + 255) & ~size_t(255);
        return r;
    };
    const size_t o_c1t = take(C1_B_BYTES);
    const size_t o_c2w = take(2 * (size_t)CST * CONV_K), o_c2b = take(4 * CST);
    const size_t o_c3w = take(2 * (size_t)CST * CONV_K), o_c3b = take(4 * CST);
    const size_t o_cow = take(2 * (size_t)D * CST * 16);
    // per layer: ln1 g/b, ln2 g/b, bqkv, bo, b1, b2 | wqkv, wo, w1, w2
    std::vector<size_t> lo(L * 12);
    for (int l = 0; l < L; l++) {
        size_t *L12 = &lo[l * 12];
        L12[0] = take(4 * D); L12[1] = take(4 * D); L12[2] = take(4 * D); L12[3] = take(4 * D);
        L12[5] = take(4 * DQKV); L12[7] = take(4 * D); L12[9] = take(4 * DFF); L12[11] = take(4 * D);
    }
    size_t big_off = 0;  // offsets inside the matrix part, rebased below
    auto take_big = [&](size_t b) {
        size_t r = big_off;
        big_off += (b + 255) & ~size_t(255);
        return r;
    };
    for (int l = 0; l < L; l++) {
        size_t *L12 = &lo[l * 12];
        L12[4] = take_big(2 * (size_t)DQKV * D);
        L12[6] = take_big(2 * (size_t)D * D);
        L12[8] = take_big(2 * (size_t)DFF * D);
        L12[10] = take_big(2 * (size_t)D * DFF);
    }
    HeadOff o_head = head_take(take, take_big);
    const size_t o_pos = take(4 * (size_t)CHUNK_TOKENS * D);
    const size_t o_mel4 = take(sizeof(Mel4Tab));
    const size_t small_total = off;
    for (int l = 0; l < L; l++)
        for (int i : {4, 6, 8, 10}) lo[l * 12 + i] += small_total;
    o_head.p1 += small_total;
    o_head.p2 += small_total;
    o_head.gu += small_total;
    o_head.wd += small_total;
    const size_t wtotal = small_total + big_off;

    std::vector<uint8_t> pk(wtotal, 0);
    auto F32 = [&](size_t o) { return reinterpret_cast<float *>(pk.data() + o); };
    auto U16 = [&](size_t o) { return reinterpret_cast<uint16_t *>(pk.data() + o); };
    const uint16_t *p = src;
    // conv1 [480][1][3][3] and its bias -> the K-major B operand of conv1_tc_kernel:
    // row c = [w(c, tap 0..8), w(c, tap 0..8), b(c), 0 ...] (64 bf16, tap = 3 kf + kt),
    // its 16-byte chunks swizzled by the row's position in its 8-row group
    {
        uint16_t *dst = U16(o_c1t);
        for (int c = 0; c < CST; c++) {
            uint16_t row[64] = {};
            for (int tap = 0; tap < 9; tap++) row[tap] = row[9 + tap] = p[c * 9 + tap];
            row[18] = p[CST * 9 + c];
            for (int k = 0; k < 64; k++) dst[c * 64 + (((k >> 3) ^ (c & 7)) << 3) + (k & 7)] = row[k];
        }
    }
    p += CST * 9 + CST;
    // conv2/conv3 [o][c][kf][kt] -> [o][(kf*3+kt)*512 + c]
    for (int which = 0; which < 2; which++) {
        uint16_t *dst = U16(which == 0 ? o_c2w : o_c3w);
        for (int o = 0; o < CST; o++)
            for (int c = 0; c < CST; c++)
                for (int tap = 0; tap < 9; tap++) dst[(size_t)o * CONV_K + tap * 512 + c] = p[((size_t)o * CST + c) * 9 + tap];
        p += (size_t)CST * CST * 9;
        float *b = F32(which == 0 ? o_c2b : o_c3b);
        for (int i = 0; i < CST; i++) b[i] = bf16_bits_to_float(p[i]);
        p += CST;
    }
    // conv_out [1280][c*16+f] -> [1280][f*480+c] (NHWC conv3 output rows)
    {
        uint16_t *dst = U16(o_cow);
        for (int o = 0; o < D; o++)
            for (int c = 0; c < CST; c++)
                for (int f = 0; f < 16; f++) dst[(size_t)o * 7680 + f * CST + c] = p[(size_t)o * 7680 + c * 16 + f];
        p += (size_t)D * 7680;
    }
    h->layers.resize(L);
    for (int l = 0; l < L; l++) {
        const size_t *L12 = &lo[l * 12];
        const size_t ln1g = L12[0], ln1b = L12[1], ln2g = L12[2], ln2b = L12[3], wqkv = L12[4], bqkv = L12[5];
        const size_t wo = L12[6], bo = L12[7], w1 = L12[8], b1 = L12[9], w2 = L12[10], b2 = L12[11];
        for (int i = 0; i < D; i++) F32(ln1g)[i] = bf16_bits_to_float(p[i]);
        p += D;
        for (int i = 0; i < D; i++) F32(ln1b)[i] = bf16_bits_to_float(p[i]);
        p += D;
        for (int part = 0; part < 3; part++) {  // q, k, v -> rows part*1280 .. of wqkv
            std::memcpy(U16(wqkv) + (size_t)part * D * D, p, 2 * (size_t)D * D);
            p += (size_t)D * D;
            for (int i = 0; i < D; i++) F32(bqkv)[part * D + i] = bf16_bits_to_float(p[i]);
            p += D;
        }
        std::memcpy(U16(wo), p, 2 * (size_t)D * D);
        p += (size_t)D * D;
        for (int i = 0; i < D; i++) F32(bo)[i] = bf16_bits_to_float(p[i]);
        p += D;
        for (int i = 0; i < D; i++) F32(ln2g)[i] = bf16_bits_to_float(p[i]);
        p += D;
        for (int i = 0; i < D; i++) F32(ln2b)[i] = bf16_bits_to_float(p[i]);
        p += D;
        std::memcpy(U16(w1), p, 2 * (size_t)DFF * D);
        p += (size_t)DFF * D;
        for (int i = 0; i < DFF; i++) F32(b1)[i] = bf16_bits_to_float(p[i]);
        p += DFF;
        std::memcpy(U16(w2), p, 2 * (size_t)D * DFF);
        p += (size_t)D * DFF;
        for (int i = 0; i < D; i++) F32(b2)[i] = bf16_bits_to_float(p[i]);
        p += D;
    }
    p = head_pack(o_head, pk.data(), p);
    if (p - src != count) return bail(MOSS_ENC_ERR_INVALID_ARG);
    // sinusoidal positions 0..99: 640 sin channels then 640 cos channels,
    // inv_timescale_i = exp(-i ln(10000) / 639)
    for (int t = 0; t < CHUNK_TOKENS; t++)
        for (int i = 0; i < D / 2; i++) {
            const double inv = std::exp(-(double)i * std::log(10000.0) / (D / 2 - 1));
            F32(o_pos)[t * D + i] = (float)std::sin(t * inv);
            F32(o_pos)[t * D + D / 2 + i] = (float)std::cos(t * inv);
        }
    {
        MelTables mt;
        if (!build_mel_tables(&mt) || !build_mel4_tab(mt, reinterpret_cast<Mel4Tab *>(pk.data() + o_mel4)))
            return bail(MOSS_ENC_ERR_INVALID_ARG);
    }

    // ---- 4-bit handles: codes and scales of every linear layer's matrix
    // (proj1/proj2 are stored [W | W] along K: W is quantised once)
    h->q4 = cfg->weight_bits == 4;
    struct QSrc {
        size_t bf_off;  // bf16 matrix in pk, rows of `stride` elements
        int n, kq, stride;
        size_t q_off, s_off;
    };
    std::vector<QSrc> qs;
    std::vector<uint8_t> qk;
    if (h->q4) {
        size_t qoff = 0;
        auto add = [&](size_t bf_off, int n, int kq, int stride) {
            QSrc q{bf_off, n, kq, stride, 0, 0};
            q.q_off = qoff;
            qoff += ((size_t)n * kq / 2 + 255) & ~size_t(255);
            q.s_off = qoff;
            qoff += ((size_t)n * (kq / 128) * 4 + 255) & ~size_t(255);
            qs.push_back(q);
        };
        for (int l = 0; l < L; l++) {
            const size_t *L12 = &lo[l * 12];
            add(L12[4], DQKV, D, D);
            add(L12[6], D, D, D);
            add(L12[8], DFF, D, D);
            add(L12[10], D, DFF, DFF);
        }
        add(o_head.p1, D, D, 2 * D);
        add(o_head.p2, DOUT, D, 2 * D);
        add(o_head.gu, 2 * DADP, DOUT, DOUT);
        add(o_head.wd, DOUT, DADP, DADP);
        qk.assign(qoff, 0);
        quantise_all(pk.data(), qk.data(), qs.data(), qs.size());
    }

    // ---- FP8 handles: q/k/v and fc1 as e4m3 per output channel, written over
    // their bf16 slots (codes [N][K], then the scales [N] at the next 256 bytes)
    h->fp8 = cfg->fp8 == 1;
    if (h->fp8) {
        std::vector<std::thread> pool;
        for (int l = 0; l < L; l++)
            for (int which = 0; which < 2; which++) {
                const size_t o = lo[l * 12 + (which == 0 ? 4 : 8)];
                const int n = which == 0 ? DQKV : DFF;
                pool.emplace_back([&pk, o, n]() { quantise_e4m3_rows(pk.data() + o, n, D); });
            }
        for (auto &th : pool) th.join();
    }
    // ---- NVFP4 handles: q/k/v (a g each) and fc1 as NVFP4 over their bf16 slots
    h->nvfp4 = cfg->nvfp4 == 1;
    if (h->nvfp4) {
        std::vector<std::thread> pool;
        for (int l = 0; l < L; l++)
            for (int which = 0; which < 2; which++) {
                const size_t o = lo[l * 12 + (which == 0 ? 4 : 8)];
                const int n = which == 0 ? DQKV : DFF, parts = which == 0 ? 3 : 1;
                pool.emplace_back([&pk, o, n, parts]() { quantise_nvfp4(pk.data() + o, n, D, parts); });
            }
        for (auto &th : pool) th.join();
    }
    const size_t upload = h->q4 ? small_total : wtotal;
    if (cudaMalloc(&h->wmem, upload) != cudaSuccess) return bail(MOSS_ENC_ERR_OOM);
    if (cudaMemcpy(h->wmem, pk.data(), upload, cudaMemcpyHostToDevice) != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);
    uint8_t *Q = nullptr;
    if (h->q4) {
        if (cudaMalloc(&h->qmem, qk.size()) != cudaSuccess) return bail(MOSS_ENC_ERR_OOM);
        if (cudaMemcpy(h->qmem, qk.data(), qk.size(), cudaMemcpyHostToDevice) != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);
        Q = static_cast<uint8_t *>(h->qmem);
    }
    auto qw = [&](size_t i) {
        QW w;
        w.codes = Q + qs[i].q_off;
        w.scales = reinterpret_cast<const float *>(Q + qs[i].s_off);
        w.kq = qs[i].kq;
        return w;
    };
    uint8_t *W = static_cast<uint8_t *>(h->wmem);
    // bf16 matrices exist on the device only for bf16 handles
    auto big = [&](size_t o) -> bf16 * { return h->q4 ? nullptr : (bf16 *)(W + o); };
    h->conv1_wt = (const uint4 *)(W + o_c1t);
    h->conv2_w = (bf16 *)(W + o_c2w);
    h->conv2_b = (float *)(W + o_c2b);
    h->conv3_w = (bf16 *)(W + o_c3w);
    h->conv3_b = (float *)(W + o_c3b);
    h->conv_out_w = (bf16 *)(W + o_cow);
    for (int l = 0; l < L; l++) {
        size_t *L12 = &lo[l * 12];
        LayerDev &d = h->layers[l];
        d.ln1_g = (float *)(W + L12[0]);
        d.ln1_b = (float *)(W + L12[1]);
        d.ln2_g = (float *)(W + L12[2]);
        d.ln2_b = (float *)(W + L12[3]);
        d.wqkv = big(L12[4]);
        d.bqkv = (float *)(W + L12[5]);
        d.wo = big(L12[6]);
        d.bo = (float *)(W + L12[7]);
        d.w1 = big(L12[8]);
        d.b1 = (float *)(W + L12[9]);
        d.w2 = big(L12[10]);
        d.b2 = (float *)(W + L12[11]);
        if (h->nvfp4) {
            d.wqkv = d.w1 = nullptr;
            d.wqkv4 = W + L12[4];
            d.sqkv4 = W + L12[4] + nvf4_sf_off(DQKV, D);
            d.gqkv4 = (const float *)(W + L12[4] + nvf4_g_off(DQKV, D));
            d.w14 = W + L12[8];
            d.s14 = W + L12[8] + nvf4_sf_off(DFF, D);
            d.g14 = (const float *)(W + L12[8] + nvf4_g_off(DFF, D));
        }
        if (h->fp8) {
            d.wqkv = d.w1 = nullptr;
            d.wqkv8 = W + L12[4];
            d.sqkv = (const float *)(W + L12[4] + f8_scale_off(DQKV, D));
            d.w18 = W + L12[8];
            d.s1 = (const float *)(W + L12[8] + f8_scale_off(DFF, D));
        }
        if (h->q4) {
            d.qqkv = qw(4 * l);
            d.qo = qw(4 * l + 1);
            d.q1 = qw(4 * l + 2);
            d.q2 = qw(4 * l + 3);
        }
    }
    h->head = head_bind(o_head, W);
    if (h->q4) {
        h->head.wp1 = h->head.wp2 = h->head.wgu = h->head.wd = nullptr;
        h->head.qp1 = qw(4 * L);
        h->head.qp2 = qw(4 * L + 1);
        h->head.qgu = qw(4 * L + 2);
        h->head.qd = qw(4 * L + 3);
    }
    h->pos = (float *)(W + o_pos);
    h->mel4_tab = (Mel4Tab *)(W + o_mel4);

    // ---- workspace
    h->max_tokens = cfg->max_samples / 1280 + cfg->max_clips + 1;
    h->max_chunks = cfg->max_samples / CHUNK_SAMPLES + cfg->max_clips + 1;
    // A 4-bit handle is the memory-saving configuration: it also runs the conv
    // stem in groups of 4 chunks (a group's conv1 activations, 24.6 MB per
    // chunk, dominate the workspace of a small handle).
    h->stem_group = (int)std::min<int64_t>(h->q4 ? 4 : STEM_GROUP_DEFAULT, h->max_chunks);
    const int64_t T = h->max_tokens, G = h->stem_group;
    off = 0;
    const size_t w_mel = take(4 * (size_t)h->max_chunks * CHUNK_FRAMES * 128);
    const size_t w_c1 = take(2 * (size_t)G * 400 * 64 * CST);
    const size_t w_c2 = take(2 * (size_t)G * 6400 * CST);
    const size_t w_c3 = take(2 * (size_t)G * 1600 * CST);
    const size_t w_X = take(4 * (size_t)T * D);
    const size_t w_xn = take(2 * (size_t)T * 2 * D);
    const size_t w_qkv = take(2 * (size_t)T * DQKV);
    const size_t w_at = take(2 * (size_t)T * D);
    const size_t w_ffn = take(2 * (size_t)T * DFF);
    const size_t w_hb = take(2 * (size_t)T * 2 * D);
    const size_t w_h2 = take(2 * (size_t)T * DOUT);
    const size_t w_gu = take(2 * (size_t)T * DADP);
    const size_t w_gm = take(4 * (size_t)cfg->max_clips);
    const size_t w_err = take(256);
    const size_t w_pcm = take(4 * (size_t)cfg->max_samples);
    const size_t w_out = take(4 * (size_t)T * DOUT);
    // 4-bit handles: one linear layer's matrix expanded to bf16 (the largest is
    // the adapter's interleaved gate/up, 16384 x 2048)
    const size_t w_qs = h->q4 ? take(2 * (size_t)2 * DADP * DOUT) : 0;
    const size_t w_rs = take(4 * (size_t)T);
    const size_t w_sf4 = h->nvfp4 ? take((size_t)(T / 128 + 1) * 20 * 512) : 0;  // NVFP4 activation scale atoms
    if (cudaMalloc(&h->ws, off) != cudaSuccess) return bail(MOSS_ENC_ERR_OOM);
    uint8_t *S = static_cast<uint8_t *>(h->ws);
    h->mel_raw = (float *)(S + w_mel);
    h->c1out = (bf16 *)(S + w_c1);
    h->c2out = (bf16 *)(S + w_c2);
    h->c3out = (bf16 *)(S + w_c3);
    h->X = (float *)(S + w_X);
    h->xn = (bf16 *)(S + w_xn);
    h->qkv = (bf16 *)(S + w_qkv);
    h->attn = (bf16 *)(S + w_at);
    h->ffn = (bf16 *)(S + w_ffn);
    h->hb = (bf16 *)(S + w_hb);
    h->h2 = (bf16 *)(S + w_h2);
    h->gu = (bf16 *)(S + w_gu);
    h->gmax_ord = (int *)(S + w_gm);
    h->err = (int *)(S + w_err);
    h->pcm_stage = (float *)(S + w_pcm);
    h->out_stage = (void *)(S + w_out);
    h->qscratch = h->q4 ? (bf16 *)(S + w_qs) : nullptr;
    h->row_scale = (float *)(S + w_rs);
    h->sfa4 = h->nvfp4 ? S + w_sf4 : nullptr;
    if (cudaMemset(h->err, 0, 256) != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);

    const TabLayout tl = tab_layout(cfg->max_clips, h->max_chunks);
    h->tab_bytes = tl.total;
    if (cudaMalloc(&h->d_tab, tl.total) != cudaSuccess) return bail(MOSS_ENC_ERR_OOM);
    if (cudaMalloc(&h->d_tab_graph, tl.total) != cudaSuccess) return bail(MOSS_ENC_ERR_OOM);
    if (cudaMallocHost(&h->h_tab_ring, tl.total * moss_enc::TAB_SLOTS) != cudaSuccess) return bail(MOSS_ENC_ERR_OOM);
    h->h_tab = h->h_tab_ring;
    for (cudaEvent_t &e : h->tab_event)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);
    if (cudaDeviceSynchronize() != cudaSuccess) return bail(MOSS_ENC_ERR_CUDA);
    *out = h;
    return MOSS_ENC_OK;
}

extern "C" moss_enc_status moss_enc_set_stream(moss_enc *h, void *stream)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    h->stream = (cudaStream_t)stream;
    return MOSS_ENC_OK;
}

extern "C" moss_enc_status moss_enc_synchronize(moss_enc *h)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    CUDA_TRY(h, cudaStreamSynchronize(h->stream));
    int e = 0;
    CUDA_TRY(h, cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost));
    if (e != 0) {
        CUDA_TRY(h, cudaMemset(h->err, 0, sizeof(int)));
        return fail(h, MOSS_ENC_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait timed out");
    }
    return MOSS_ENC_OK;
}

// --------------------------------------------------------- per-call tables

// A call's tables are written into the next host staging area of the ring
// (h->h_tab), once the copy that last read that area has run (not waited
// for while a stream is being captured).
static moss_enc_status tab_begin(moss_enc *h)
{
    h->tab_slot = (h->tab_slot + 1) % moss_enc::TAB_SLOTS;
    h->h_tab = static_cast<uint8_t *>(h->h_tab_ring) + (size_t)h->tab_slot * h->tab_bytes;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    CUDA_TRY(h, cudaStreamIsCapturing(h->stream, &cs));
    if (cs == cudaStreamCaptureStatusNone) CUDA_TRY(h, cudaEventSynchronize(h->tab_event[h->tab_slot]));
    return MOSS_ENC_OK;
}

// Copy the current tables to dst (the device tables of launch-by-launch
// calls, or those a captured forward graph reads), in stream order: the copy
// runs after every earlier kernel on the stream has finished with them.
static moss_enc_status tab_upload(moss_enc *h, void *dst = nullptr)
{
    CUDA_TRY(h, cudaMemcpyAsync(dst ? dst : h->d_tab, h->h_tab, h->tab_bytes, cudaMemcpyHostToDevice, h->stream));
    CUDA_TRY(h, cudaEventRecord(h->tab_event[h->tab_slot], h->stream));
    return MOSS_ENC_OK;
}


static moss_enc_status launch_logmel(moss_enc *h, const MelClip *d_clips, int n_clips, int64_t max_frames,
                                     float *out, int write_out, int64_t total_frames)
{
    if (n_clips <= 0 || max_frames <= 0) return MOSS_ENC_OK;
    for (int c0 = 0; c0 < n_clips; c0 += MEL_MAX_CLIPS) {
        const int nc = std::min(MEL_MAX_CLIPS, n_clips - c0);
        const int64_t blocks = (int64_t)nc * ((max_frames + MEL4_FRAMES - 1) / MEL4_FRAMES);  // upper bound
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(blocks, 4 * h->num_sms));
        Launch L(h, write_out ? "logmel" : "logmel_max", 0.0,
                 c0 == 0 ? 4.0 * 160 * (double)total_frames + (write_out ? 512.0 * total_frames : 0.0) : 0.0);
        CUDA_TRY(h, launch_k(h, logmel4_kernel, dim3(grid), dim3(MEL4_THREADS), sizeof(Mel4Smem), d_clips + c0, nc,
                             (const Mel4Tab *)h->mel4_tab, out, h->gmax_ord, write_out));
    }
    return MOSS_ENC_OK;
}

// ------------------------------------------------------------------ logmel

extern "C" moss_enc_status moss_enc_log_max(moss_enc *h, const float *pcm, int64_t n_samples, float *out)
{
    if (!h || !pcm || !out || n_samples < 0) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad argument");
    if (n_samples / HOP > INT32_MAX) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "clip too long");
    TRY(tab_begin(h));
    const TabLayout tl = tab_layout(h->cfg.max_clips, h->max_chunks);
    uint8_t *H = static_cast<uint8_t *>(h->h_tab);
    const float **src = reinterpret_cast<const float **>(H + tl.logmax_src);
    src[0] = nullptr;
    MelClip *mc = reinterpret_cast<MelClip *>(H + tl.clips_max);
    mc[0] = MelClip{pcm, (long long)n_samples, 0, 0, (int)(n_samples / HOP), 0, 0};
    TRY(tab_upload(h));
    uint8_t *Dt = static_cast<uint8_t *>(h->d_tab);
    {
        Launch Lk(h, "gmax", 0.0, 0.0);
        gmax_init_kernel<<<1, 32, 0, h->stream>>>(h->gmax_ord, reinterpret_cast<const float *const *>(Dt + tl.logmax_src), 1);
    }
    CUDA_TRY(h, cudaGetLastError());
    TRY(launch_logmel(h, reinterpret_cast<const MelClip *>(Dt + tl.clips_max), 1, n_samples / HOP, nullptr, 0, n_samples / HOP));
    {
        Launch Lk(h, "gmax", 0.0, 0.0);
        gmax_export_kernel<<<1, 32, 0, h->stream>>>(h->gmax_ord, out);
    }
    CUDA_TRY(h, cudaGetLastError());
    return MOSS_ENC_OK;
}

extern "C" moss_enc_status moss_enc_range_log_max(moss_enc *h, const float *pcm, int64_t n_samples, int64_t begin,
                                                  int64_t end, float *out)
{
    if (!h || !pcm || !out || n_samples < 0) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad argument");
    if (begin < 0 || end < begin || end > n_samples || begin % HOP != 0 || (end != n_samples && end % HOP != 0))
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad range");
    if (n_samples / HOP > INT32_MAX) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "clip too long");
    const int64_t f_begin = begin / HOP, f_end = end == n_samples ? n_samples / HOP : end / HOP;
    TRY(tab_begin(h));
    const TabLayout tl = tab_layout(h->cfg.max_clips, h->max_chunks);
    uint8_t *H = static_cast<uint8_t *>(h->h_tab);
    reinterpret_cast<const float **>(H + tl.logmax_src)[0] = nullptr;
    MelClip *mc = reinterpret_cast<MelClip *>(H + tl.clips_max);
    mc[0] = MelClip{pcm, (long long)n_samples, 0, (int)f_begin, (int)f_end, 0, 0};
    TRY(tab_upload(h));
    uint8_t *Dt = static_cast<uint8_t *>(h->d_tab);
    {
        Launch Lk(h, "gmax", 0.0, 0.0);
        gmax_init_kernel<<<1, 32, 0, h->stream>>>(h->gmax_ord, reinterpret_cast<const float *const *>(Dt + tl.logmax_src), 1);
    }
    CUDA_TRY(h, cudaGetLastError());
    TRY(launch_logmel(h, reinterpret_cast<const MelClip *>(Dt + tl.clips_max), 1, f_end - f_begin, nullptr, 0,
                      f_end - f_begin));
    {
        Launch Lk(h, "gmax", 0.0, 0.0);
        gmax_export_kernel<<<1, 32, 0, h->stream>>>(h->gmax_ord, out);
    }
    CUDA_TRY(h, cudaGetLastError());
    return MOSS_ENC_OK;
}

extern "C" moss_enc_status moss_enc_logmel(moss_enc *h, const moss_enc_clip *clip, float *mel_out,
                                           int64_t *n_frames, float *log_max_out)
{
    if (!h || !clip || !clip->pcm) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad argument");
    ClipPlan pl;
    if (!plan_clip(clip->n_samples, clip->begin, clip->end, &pl)) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad range");
    if (pl.F > INT32_MAX) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "clip too long");
    if (clip->end - clip->begin > h->cfg.max_samples) return fail(h, MOSS_ENC_ERR_CAPACITY, "range exceeds max_samples");
    const int64_t nf = pl.f_end - pl.f_begin;
    if (n_frames) *n_frames = nf;
    if (nf > 0 && !mel_out) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "mel_out is null");
    const bool whole = pl.f_begin == 0 && pl.f_end == pl.F;
    TRY(tab_begin(h));
    const TabLayout tl = tab_layout(h->cfg.max_clips, h->max_chunks);
    uint8_t *H = static_cast<uint8_t *>(h->h_tab);
    reinterpret_cast<const float **>(H + tl.logmax_src)[0] = clip->log_max;
    MelClip *mm = reinterpret_cast<MelClip *>(H + tl.clips_main);
    MelClip *mx = reinterpret_cast<MelClip *>(H + tl.clips_max);
    const bool own_max = clip->log_max == nullptr;
    mm[0] = MelClip{clip->pcm, (long long)pl.n, 0, (int)pl.f_begin, (int)pl.f_end, own_max && whole ? 0 : -1, 0};
    mx[0] = MelClip{clip->pcm, (long long)pl.n, 0, 0, (int)pl.F, 0, 0};
    TRY(tab_upload(h));
    uint8_t *Dt = static_cast<uint8_t *>(h->d_tab);
    {
        Launch Lk(h, "gmax", 0.0, 0.0);
        gmax_init_kernel<<<1, 32, 0, h->stream>>>(h->gmax_ord, reinterpret_cast<const float *const *>(Dt + tl.logmax_src), 1);
    }
    CUDA_TRY(h, cudaGetLastError());
    if (own_max && !whole)
        TRY(launch_logmel(h, reinterpret_cast<const MelClip *>(Dt + tl.clips_max), 1, pl.F, nullptr, 0, pl.F));
    TRY(launch_logmel(h, reinterpret_cast<const MelClip *>(Dt + tl.clips_main), 1, nf, mel_out, 1, nf));
    if (nf > 0) {
        {
            Launch Lk(h, "mel_normalize", 0.0, 8.0 * nf * 128);
            mel_normalize_kernel<<<std::min<int64_t>(4096, (nf * 128 + 255) / 256), 256, 0, h->stream>>>(mel_out, nf * 128, h->gmax_ord);
        }
        CUDA_TRY(h, cudaGetLastError());
    }
    if (log_max_out) {
        {
            Launch Lk(h, "gmax", 0.0, 0.0);
            gmax_export_kernel<<<1, 32, 0, h->stream>>>(h->gmax_ord, log_max_out);
        }
        CUDA_TRY(h, cudaGetLastError());
    }
    return MOSS_ENC_OK;
}

// ----------------------------------------------------------------- forward

// Host-side result of planning one forward: counts and the per-group conv
// tile lists (the tables themselves sit in the staging buffer).
struct FwdPlan {
    int n_clips = 0;
    int64_t n_chunks = 0, T = 0;
    int n_max_pass = 0;
    int64_t max_clip_frames = 0, max_range_frames = 0, max_pass_frames = 0, range_frames = 0;
    const StemChunk *sc = nullptr;
    const int2 *ct = nullptr;
    std::vector<int> g_off2, g_n2, g_off3, g_n3;
};

// Shape of a forward request for graph reuse: every host-side value the
// launch sequence depends on (grids, GEMM sizes, the stem groups' tile
// counts) and the tap outputs.  Two requests of one shape launch the same
// kernels with the same parameters; what differs between them (the PCM
// pointers and ranges, the per-chunk tables) is read from the device tables.
static std::vector<uint8_t> shape_key(const FwdPlan &P, void *const *tap_out, int n_taps)
{
    const int nt = tap_out ? n_taps : 0;
    std::vector<int64_t> v = {P.n_clips, P.n_chunks, P.T, P.n_max_pass, P.max_clip_frames, P.max_range_frames, nt,
                              (int64_t)P.g_n2.size()};
    for (size_t g = 0; g < P.g_n2.size(); g++) {
        v.push_back(P.g_n2[g]);
        v.push_back(P.g_n3[g]);
    }
    for (int t = 0; t < nt; t++) v.push_back((int64_t)reinterpret_cast<uintptr_t>(tap_out[t]));
    std::vector<uint8_t> k(v.size() * sizeof(int64_t));
    std::memcpy(k.data(), v.data(), k.size());
    return k;
}

// 4-bit handles.  A GEMM of one 256-row tile expands the codes in shared
// memory as it goes (gemm2q); a larger one would expand the same matrix once
// per 256-row tile, so the matrices are expanded once per forward, into the
// workspace's scratch, by a bandwidth-bound kernel, and the bf16 GEMMs run on
// them (same values, same arithmetic).  q4_expand launches one expansion of
// up to four matrices (mats[i] -> outs[i], rows repeated reps[i] times along
// k).  A GEMM that starts its weight loads before waiting on earlier kernels
// is safe behind it as long as one kernel that waits before letting its
// dependents start (LayerNorm) lies between them; right after it, the GEMM is
// launched without overlap (after_expand).
static moss_enc_status q4_expand(moss_enc *h, const QW *const *mats, const int *n, const int *reps, bf16 *const *outs,
                                 int count, bool after_expand)
{
    Q4Jobs J{};
    J.count = count;
    double bytes = 0.0;
    for (int i = 0; i < count; i++) {
        J.j[i] = Q4Job{mats[i]->codes, mats[i]->scales, outs[i], n[i], mats[i]->kq, reps[i], J.items};
        J.items += (long long)n[i] * (mats[i]->kq / 32);
        bytes += 0.5 * n[i] * (double)mats[i]->kq + 4.0 * n[i] * (mats[i]->kq / 128) + 2.0 * n[i] * reps[i] * (double)mats[i]->kq;
    }
    const int grid = (int)std::min<long long>((J.items + 255) / 256, 8LL * h->num_sms);
    Launch L(h, "q4_expand", 0.0, bytes);
    CUDA_TRY(h, launch_k(h, q4_expand_kernel, dim3(grid), dim3(256), 0, J));
    if (after_expand) h->pdl_skip_once = true;
    return MOSS_ENC_OK;
}

// One matrix into the scratch, for the GEMM launched next.
static const bf16 *q4_expand_one(moss_enc *h, const QW &q, int n, int reps, moss_enc_status *st)
{
    const QW *m = &q;
    bf16 *o = h->qscratch;
    *st = q4_expand(h, &m, &n, &reps, &o, 1, true);
    return h->qscratch;
}

// Pair-tile width for an M x N x K GEMM among the candidates `order`: the one
// whose busiest SM pair has the fewest output columns to compute (pair tiles
// of one width are spread evenly over the pairs), with 128-wide tiles counted
// 1.5 times for long mainloops (K >= 4096), where an N = 128 MMA's lower rate
// dominates (measured 2358 against 3707-3811 MACs per clock and SM for N of
// 256 or 160).  Ties go to the earlier candidate.  The tile width never
// changes an output element's arithmetic.
static int pick_width(const moss_enc *h, int64_t M, int N, int K, const int *order, int n)
{
    const int64_t m = (M + 255) / 256, pairs = std::max(1, h->num_sms / 2);
    int best = order[0];
    double best_cost = 1e300;
    for (int i = 0; i < n; i++) {
        const int64_t tiles = m * (N / order[i]);
        const double cost = (double)((tiles + pairs - 1) / pairs) * order[i] * (order[i] == 128 && K >= 4096 ? 1.5 : 1.0);
        if (cost < best_cost) {
            best_cost = cost;
            best = order[i];
        }
    }
    return best;
}

// ln_post -> proj1 -> GELU -> proj2 -> SwiGLU adapter on the residual stream
// X [T][1280], with the head set W; stops after proj2 (fp32 rows) when stage
// is MOSS_ENC_STAGE_HEAD, else writes the adapter rows (cfg.out_dtype).
static moss_enc_status head_launch(moss_enc *h, const HeadDev &W, int64_t T, int stage, void *out)
{
    const int ln_grid = (int)((T + 7) / 8);
    {
        Launch Lk(h, "layernorm", 8.0 * T * D, 6.0 * T * D);
        CUDA_TRY(h, launch_k(h, layernorm1280_kernel, dim3(ln_grid), dim3(256), 0, (const float *)h->X,
                             (const float *)W.lnp_g, (const float *)W.lnp_b, h->xn, (int)T, 2 * D, 1));
    }
    // The two head GEMMs take split operands [hi | lo] (bf16 pairs that carry
    // ~16 bits) against weights repeated along K; the adapter's inputs (proj2's
    // output and the SwiGLU product) are plain bf16.  Splitting the gate/up
    // input as well doubles the adapter's largest GEMM for little: over 1196
    // rows of the 30 s clip, the 16-clip batch and the 10-min clip the final
    // rows' worst max err/rms is 0.0225 without it and 0.0194 with it, against
    // a bound of 0.03.
    // a set with 4-bit matrices: one 256-row tile takes the 4-bit GEMM (same
    // tiles, same epilogues), a larger batch expands each matrix once
    const bool q = W.qp1.codes != nullptr && T <= 256;
    const bool qx = W.qp1.codes != nullptr && T > 256;
    moss_enc_status qst = MOSS_ENC_OK;
    GemmArgs a{};
    a.bias = W.bp1;
    a.out = h->hb;
    a.ldo = 2 * D;
    a.split_off = D;
    if (q) {
        TRY((gemm2q<320, EPI_GELU_BF16>(h, "gemm_proj1", h->xn, T, 2 * D, W.qp1, D, a, D)));
    } else {
        const bf16 *B = qx ? q4_expand_one(h, W.qp1, D, 2, &qst) : W.wp1;
        TRY(qst);
        TRY((gemm2<320, EPI_GELU_BF16>(h, "gemm_proj1", h->xn, T, 2 * D, B, D, a, D)));
    }
    a.bias = W.bp2;
    const bf16 *B2 = W.wp2;
    if (qx) {
        B2 = q4_expand_one(h, W.qp2, DOUT, 2, &qst);
        TRY(qst);
    }
    if (stage == MOSS_ENC_STAGE_HEAD) {
        a.out = out;
        a.ldo = DOUT;
        a.split_off = 0;
        return q ? gemm2q<256, EPI_F32>(h, "gemm_proj2", h->hb, T, 2 * D, W.qp2, DOUT, a, D)
                 : gemm2<256, EPI_F32>(h, "gemm_proj2", h->hb, T, 2 * D, B2, DOUT, a, D);
    }
    a.out = h->h2;
    a.ldo = DOUT;
    a.split_off = 0;
    TRY((q ? gemm2q<256, EPI_BF16>(h, "gemm_proj2", h->hb, T, 2 * D, W.qp2, DOUT, a, D)
          : gemm2<256, EPI_BF16>(h, "gemm_proj2", h->hb, T, 2 * D, B2, DOUT, a, D)));
    // ---- SwiGLU adapter
    a.bias = W.bgu;
    a.out = h->gu;
    a.ldo = DADP;
    const bf16 *Bgu = W.wgu;
    if (qx) {
        Bgu = q4_expand_one(h, W.qgu, 2 * DADP, 1, &qst);
        TRY(qst);
    }
    TRY((q ? gemm2q<256, EPI_SWIGLU_BF16>(h, "gemm_gate_up", h->h2, T, DOUT, W.qgu, 2 * DADP, a)
          : gemm2<256, EPI_SWIGLU_BF16>(h, "gemm_gate_up", h->h2, T, DOUT, Bgu, 2 * DADP, a)));
    a.bias = W.bd;
    a.out = out;
    a.ldo = DOUT;
    a.split_off = 0;
    static const int down_w[2] = {256, 128};
    const bool narrow = pick_width(h, T, DOUT, DADP, down_w, 2) == 128;
    const bf16 *Bd = W.wd;
    if (qx) {
        Bd = q4_expand_one(h, W.qd, DOUT, 1, &qst);
        TRY(qst);
    }
    if (q) {
        if (h->cfg.out_dtype == MOSS_ENC_OUT_F32)
            return narrow ? gemm2q<128, EPI_F32>(h, "gemm_down", h->gu, T, DADP, W.qd, DOUT, a)
                          : gemm2q<256, EPI_F32>(h, "gemm_down", h->gu, T, DADP, W.qd, DOUT, a);
        return narrow ? gemm2q<128, EPI_BF16>(h, "gemm_down", h->gu, T, DADP, W.qd, DOUT, a)
                      : gemm2q<256, EPI_BF16>(h, "gemm_down", h->gu, T, DADP, W.qd, DOUT, a);
    }
    if (h->cfg.out_dtype == MOSS_ENC_OUT_F32)
        return narrow ? gemm2<128, EPI_F32>(h, "gemm_down", h->gu, T, DADP, Bd, DOUT, a)
                      : gemm2<256, EPI_F32>(h, "gemm_down", h->gu, T, DADP, Bd, DOUT, a);
    return narrow ? gemm2<128, EPI_BF16>(h, "gemm_down", h->gu, T, DADP, Bd, DOUT, a)
                  : gemm2<256, EPI_BF16>(h, "gemm_down", h->gu, T, DADP, Bd, DOUT, a);
}

static moss_enc_status forward_launch(moss_enc *h, const FwdPlan &P, uint8_t *Dt, int stage, void *out,
                                     void *const *tap_out)
{
    const TabLayout tl = tab_layout(h->cfg.max_clips, h->max_chunks);
    const int n_clips = P.n_clips;
    const int64_t n_chunks = P.n_chunks, T = P.T;
    const int n_max_pass = P.n_max_pass;
    const int64_t max_clip_frames = P.max_clip_frames, max_range_frames = P.max_range_frames;
    const int64_t max_pass_frames = P.max_pass_frames, range_frames = P.range_frames;
    const StemChunk *sc = P.sc;
    const int2 *ct = P.ct;
    const std::vector<int> &g_off2 = P.g_off2, &g_n2 = P.g_n2, &g_off3 = P.g_off3, &g_n3 = P.g_n3;
    const StemChunk *d_chunks = reinterpret_cast<const StemChunk *>(Dt + tl.chunks);
    const int *d_t2 = reinterpret_cast<const int *>(Dt + tl.tiles2);
    const int *d_t3 = reinterpret_cast<const int *>(Dt + tl.tiles3);
    const int2 *d_ct = reinterpret_cast<const int2 *>(Dt + tl.chunk_tok);

    // ---- log-mel (raw) and per-clip maxima
    {
        Launch Lk(h, "gmax", 0.0, 0.0);
        CUDA_TRY(h, launch_k(h, gmax_init_kernel, dim3((n_clips + 127) / 128), dim3(128), 0, h->gmax_ord,
                             reinterpret_cast<const float *const *>(Dt + tl.logmax_src), n_clips));
    }
    if (n_max_pass > 0)
        TRY(launch_logmel(h, reinterpret_cast<const MelClip *>(Dt + tl.clips_max), n_max_pass, max_clip_frames, nullptr, 0, max_pass_frames));
    TRY(launch_logmel(h, reinterpret_cast<const MelClip *>(Dt + tl.clips_main), n_clips, max_range_frames, h->mel_raw, 1, range_frames));

    // ---- conv stem, in groups of chunks; only tiles inside the receptive
    // field of each chunk's tokens are computed
    for (int64_t g0 = 0, gi = 0; g0 < n_chunks; g0 += h->stem_group, gi++) {
        const int gc = (int)std::min<int64_t>(h->stem_group, n_chunks - g0);
        {
            double px = 0.0;
            for (int j = 0; j < gc; j++) px += 64.0 * sc[g0 + j].t1_lim;
            int tiles = 0;  // 128-pixel tiles (two time steps) inside the receptive fields
            for (int j = 0; j < gc; j++) tiles += (sc[g0 + j].t1_lim + 1) / 2;
            Launch L1(h, "conv1", 2.0 * 9 * CST * px, 2.0 * CST * px + 4.0 * 128 * 2 * px / 64.0);
            CUtensorMap tm_c1;  // conv1 output rows [chunk][t][f] x 480 channels: boxes of 80 x 32
            if (!tmap_2d(&tm_c1, h->c1out, CST, (uint64_t)gc * 400 * 64, 2 * CST, 80, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
                return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (conv1 output)");
            CUDA_TRY(h, launch_k(h, conv1_tc_kernel, dim3(std::max(1, std::min(tiles, h->num_sms))), dim3(C1_THREADS),
                                 C1_SMEM, (const float *)h->mel_raw, d_chunks + g0, gc, (const int *)h->gmax_ord,
                                 h->conv1_wt, tm_c1, h->err));
        }
        TRY(gemm_conv(h, "gemm_conv2", h->c1out, gc, 400, 64, d_t2 + g_off2[gi], g_n2[gi], h->conv2_w, h->conv2_b,
                      h->c2out));
        TRY(gemm_conv(h, "gemm_conv3", h->c2out, gc, 200, 32, d_t3 + g_off3[gi], g_n3[gi], h->conv3_w, h->conv3_b,
                      h->c3out));
        GemmArgs co{};
        co.out = h->X;
        co.ldo = D;
        co.pos = h->pos;
        co.chunk_tok = d_ct + g0;
        TRY((gemm2<320, EPI_CONVOUT_F32>(h, "gemm_conv_out", h->c3out, (int64_t)gc * 100, 7680, h->conv_out_w, D, co)));
    }
    if (stage == MOSS_ENC_STAGE_STEM) {
        CUDA_TRY(h, cudaMemcpyAsync(out, h->X, sizeof(float) * T * D, cudaMemcpyDeviceToDevice, h->stream));
        return MOSS_ENC_OK;
    }

    // ---- Transformer layers
    const int ln_grid = (int)((T + 7) / 8);
    double attn_pairs = 0.0;  // query-key pairs inside windows
    for (int64_t c = 0; c < n_chunks; c++) attn_pairs += (double)ct[c].y * ct[c].y;
    static_assert(CHUNK_TOKENS <= ATTN_ROWS, "a window must fit the attention kernel's slices");
    CUtensorMap tm_qkv;  // Q, K, V slices of one window and head: ATTN_ROWS rows x 64
    if (!tmap_2d(&tm_qkv, h->qkv, (uint64_t)DQKV, (uint64_t)T, (uint64_t)DQKV * 2, 64, ATTN_ROWS))
        return fail(h, MOSS_ENC_ERR_CUDA, "cuTensorMapEncodeTiled failed (qkv)");
    // Tile width of the N = 1280 residual GEMMs (out-proj, FC2): the one whose
    // busiest SM pair has the fewest output columns to compute (the pair
    // tiles of one width are spread evenly over the pairs), ties broken
    // toward 320 for the long K = 5120 mainloop (wider tiles need the least
    // operand bandwidth per MMA) and toward 160 for K = 1280 (two tiles per
    // pair let one tile's epilogue run under the other's mainloop).  The tile
    // width does not change any output element's arithmetic, so a clip's rows
    // are the same at every batch size.
    // 4-bit handles: a batch of one 256-row tile takes the 4-bit GEMM, a
    // larger one expands each matrix once into the scratch (q4_expand)
    const bool qf = h->q4 && T <= 256, qx = h->q4 && T > 256;
    auto resid_gemm = [&](const char *name, const bf16 *Ain, int K, const bf16 *W, const QW &Wq,
                          GemmArgs a) -> moss_enc_status {
        static const int long_k[3] = {320, 160, 128}, short_k[3] = {160, 128, 320};
        const int bn = pick_width(h, T, D, K, K > D ? long_k : short_k, 3);
        if (qf) {
            if (bn == 128) return gemm2q<128, EPI_RESID_F32>(h, name, Ain, T, K, Wq, D, a);
            if (bn == 160) return gemm2q<160, EPI_RESID_F32>(h, name, Ain, T, K, Wq, D, a);
            return gemm2q<320, EPI_RESID_F32>(h, name, Ain, T, K, Wq, D, a);
        }
        switch (bn) {
        case 128: return gemm2<128, EPI_RESID_F32>(h, name, Ain, T, K, W, D, a, 0, 2);
        case 160: return gemm2<160, EPI_RESID_F32>(h, name, Ain, T, K, W, D, a, 0, 2);
        default: return gemm2<320, EPI_RESID_F32>(h, name, Ain, T, K, W, D, a, 0, K == D ? 2 : 1);
        }
    };
    // 4-bit handles, larger batches: the layer's four matrices in the scratch
    bf16 *xs_qkv = h->qscratch, *xs_o = xs_qkv + (size_t)DQKV * D, *xs_1 = xs_o + (size_t)D * D,
         *xs_2 = xs_1 + (size_t)DFF * D;
    for (size_t l = 0; l < h->layers.size(); l++) {
        const LayerDev &L = h->layers[l];
        const bf16 *Wqkv = L.wqkv, *Wo = L.wo, *W1 = L.w1, *W2 = L.w2;
        if (qx) {
            // expanded before LN1, which waits on it before letting the QKV
            // GEMM start (that GEMM requests its weights before waiting)
            const QW *m[4] = {&L.qqkv, &L.qo, &L.q1, &L.q2};
            const int n[4] = {DQKV, D, DFF, D}, r[4] = {1, 1, 1, 1};
            bf16 *const o[4] = {xs_qkv, xs_o, xs_1, xs_2};
            TRY(q4_expand(h, m, n, r, o, 4, false));
            Wqkv = xs_qkv;
            Wo = xs_o;
            W1 = xs_1;
            W2 = xs_2;
        }
        uint8_t *xn8 = reinterpret_cast<uint8_t *>(h->xn);  // FP8 / NVFP4 handles: the LayerNorm rows' codes
        if (h->nvfp4) {
            Launch Lk(h, "layernorm", 8.0 * T * D, 4.0 * T * D + 0.5 * T * D + T * D / 16.0);
            CUDA_TRY(h, launch_k(h, nvf4_rows1280_kernel<true>, dim3(ln_grid), dim3(256), 0, (const float *)h->X,
                                 L.ln1_g, L.ln1_b, xn8, h->sfa4, h->row_scale, (int)T));
        } else if (h->fp8) {
            Launch Lk(h, "layernorm", 8.0 * T * D, 5.0 * T * D);
            CUDA_TRY(h, launch_k(h, layernorm1280_e4m3_kernel, dim3(ln_grid), dim3(256), 0, (const float *)h->X, L.ln1_g,
                                 L.ln1_b, xn8, h->row_scale, (int)T));
        } else {
            Launch Lk(h, "layernorm", 8.0 * T * D, 6.0 * T * D);
            CUDA_TRY(h, launch_k(h, layernorm1280_kernel, dim3(ln_grid), dim3(256), 0, (const float *)h->X, L.ln1_g, L.ln1_b,
                                 h->xn, (int)T, D, 0));
        }
        GemmArgs a{};
        a.bias = L.bqkv;
        a.out = h->qkv;
        a.ldo = DQKV;
        if (h->nvfp4) {
            a.row_scale = h->row_scale;
            a.col_scale = L.gqkv4;
            a.sfa = h->sfa4;
            a.sfb = L.sqkv4;
            TRY((gemm_nvf4<EPI_BF16>(h, "gemm_qkv", xn8, T, D, L.wqkv4, DQKV, a)));
            a.row_scale = a.col_scale = nullptr;
            a.sfa = a.sfb = nullptr;
        } else if (h->fp8) {
            a.row_scale = h->row_scale;
            a.col_scale = L.sqkv;
            if (T <= 512)
                TRY((gemm2f8<128, EPI_BF16>(h, "gemm_qkv", xn8, T, D, L.wqkv8, DQKV, a)));
            else
                TRY((gemm2f8<256, EPI_BF16>(h, "gemm_qkv", xn8, T, D, L.wqkv8, DQKV, a)));
            a.row_scale = a.col_scale = nullptr;
        } else if (qf)
            TRY((gemm2q<128, EPI_BF16>(h, "gemm_qkv", h->xn, T, D, L.qqkv, DQKV, a)));
        else if (T <= 512)  // two row tiles: 128-wide tiles (30 per row tile) keep more SMs busy than 256-wide (15)
            TRY((gemm2<128, EPI_BF16>(h, "gemm_qkv", h->xn, T, D, Wqkv, DQKV, a)));
        else
            TRY((gemm2<256, EPI_BF16>(h, "gemm_qkv", h->xn, T, D, Wqkv, DQKV, a)));
        {
            Launch Lk(h, "attention", 4.0 * 64 * 20 * attn_pairs, 2.0 * T * (DQKV + D));
            CUDA_TRY(h, launch_k(h, window_attn_tc_kernel, dim3((unsigned)n_chunks, 20), dim3(128), ATTN_TC_SMEM, tm_qkv,
                                 d_ct, h->attn, h->err));
        }
        a.bias = L.bo;
        a.out = h->X;
        a.ldo = D;
        TRY(resid_gemm("gemm_out", h->attn, D, Wo, L.qo, a));
        if (h->nvfp4) {
            Launch Lk(h, "layernorm", 8.0 * T * D, 4.0 * T * D + 0.5 * T * D + T * D / 16.0);
            CUDA_TRY(h, launch_k(h, nvf4_rows1280_kernel<true>, dim3(ln_grid), dim3(256), 0, (const float *)h->X,
                                 L.ln2_g, L.ln2_b, xn8, h->sfa4, h->row_scale, (int)T));
        } else if (h->fp8) {
            Launch Lk(h, "layernorm", 8.0 * T * D, 5.0 * T * D);
            CUDA_TRY(h, launch_k(h, layernorm1280_e4m3_kernel, dim3(ln_grid), dim3(256), 0, (const float *)h->X, L.ln2_g,
                                 L.ln2_b, xn8, h->row_scale, (int)T));
        } else {
            Launch Lk(h, "layernorm", 8.0 * T * D, 6.0 * T * D);
            CUDA_TRY(h, launch_k(h, layernorm1280_kernel, dim3(ln_grid), dim3(256), 0, (const float *)h->X, L.ln2_g, L.ln2_b,
                                 h->xn, (int)T, D, 0));
        }
        a.bias = L.b1;
        a.out = h->ffn;
        a.ldo = DFF;
        if (h->nvfp4) {
            a.row_scale = h->row_scale;
            a.col_scale = L.g14;
            a.sfa = h->sfa4;
            a.sfb = L.s14;
            TRY((gemm_nvf4<EPI_GELU_BF16>(h, "gemm_fc1", xn8, T, D, L.w14, DFF, a)));
            a.row_scale = a.col_scale = nullptr;
            a.sfa = a.sfb = nullptr;
        } else if (h->fp8) {
            a.row_scale = h->row_scale;
            a.col_scale = L.s1;
            TRY((gemm2f8<256, EPI_GELU_BF16>(h, "gemm_fc1", xn8, T, D, L.w18, DFF, a)));
            a.row_scale = a.col_scale = nullptr;
        } else
        TRY((qf ? gemm2q<256, EPI_GELU_BF16>(h, "gemm_fc1", h->xn, T, D, L.q1, DFF, a)
                : gemm2<256, EPI_GELU_BF16>(h, "gemm_fc1", h->xn, T, D, W1, DFF, a)));
        a.bias = L.b2;
        a.out = h->X;
        a.ldo = D;
        TRY(resid_gemm("gemm_fc2", h->ffn, DFF, W2, L.q2, a));
        // layer taps: this layer's hidden states through the tap's own head set
        // (xn, hb, h2 and gu are free between layers)
        if (tap_out)
            for (size_t t = 0; t < h->tap_layers.size(); t++)
                if (h->tap_layers[t] == (int)l) TRY(head_launch(h, h->tap_heads[t], T, MOSS_ENC_STAGE_ADAPTER, tap_out[t]));
    }
    if (stage == MOSS_ENC_STAGE_LAYERS) {
        CUDA_TRY(h, cudaMemcpyAsync(out, h->X, sizeof(float) * T * D, cudaMemcpyDeviceToDevice, h->stream));
        return MOSS_ENC_OK;
    }

    return head_launch(h, h->head, T, stage, out);
}

static moss_enc_status forward_impl(moss_enc *h, const moss_enc_clip *clips, int n_clips, int stage,
                                    void *out, int64_t *row_offsets, void *const *tap_out = nullptr)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (n_clips < 0 || (n_clips > 0 && !clips) || !row_offsets) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad argument");
    if (n_clips > h->cfg.max_clips) return fail(h, MOSS_ENC_ERR_CAPACITY, "too many clips");
    if (stage < MOSS_ENC_STAGE_STEM || stage > MOSS_ENC_STAGE_ADAPTER) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad stage");

    std::vector<ClipPlan> plans(n_clips);
    int64_t samples = 0, T = 0, n_chunks = 0, max_range_frames = 0, max_clip_frames = 0;
    row_offsets[0] = 0;
    for (int i = 0; i < n_clips; i++) {
        const moss_enc_clip &c = clips[i];
        if (!plan_clip(c.n_samples, c.begin, c.end, &plans[i])) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad clip range");
        if (plans[i].ntok > 0 && !c.pcm) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "null pcm");
        if (plans[i].F > INT32_MAX / 2) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "clip too long");
        plans[i].tok0 = T;
        T += plans[i].ntok;
        row_offsets[i + 1] = T;
        samples += c.end - c.begin;
        n_chunks += plans[i].c_last - plans[i].c_first;
        max_range_frames = std::max(max_range_frames, plans[i].f_end - plans[i].f_begin);
        max_clip_frames = std::max(max_clip_frames, plans[i].F);
    }
    if (samples > h->cfg.max_samples || T > h->max_tokens || n_chunks > h->max_chunks)
        return fail(h, MOSS_ENC_ERR_CAPACITY, "request exceeds the capacity set at create");
    if (T > 0 && !out) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "null output");
    if (T > 0 && tap_out)
        for (size_t t = 0; t < h->tap_layers.size(); t++)
            if (!tap_out[t]) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "null tap output");
    if (T == 0) return MOSS_ENC_OK;

    // ---- tables
    TRY(tab_begin(h));
    const TabLayout tl = tab_layout(h->cfg.max_clips, h->max_chunks);
    uint8_t *H = static_cast<uint8_t *>(h->h_tab);
    const float **lsrc = reinterpret_cast<const float **>(H + tl.logmax_src);
    MelClip *mm = reinterpret_cast<MelClip *>(H + tl.clips_main);
    MelClip *mx = reinterpret_cast<MelClip *>(H + tl.clips_max);
    StemChunk *sc = reinterpret_cast<StemChunk *>(H + tl.chunks);
    int2 *ct = reinterpret_cast<int2 *>(H + tl.chunk_tok);
    int n_max_pass = 0;
    int64_t chunk = 0, max_pass_frames = 0, range_frames = 0;
    for (int i = 0; i < n_clips; i++) {
        const ClipPlan &pl = plans[i];
        const bool whole = pl.f_begin == 0 && pl.f_end == pl.F;
        const bool own = clips[i].log_max == nullptr;
        lsrc[i] = clips[i].log_max;
        // main pass: frames [800 c_first, f_end) into rows of this clip's chunks
        const int64_t fb = pl.c_first * CHUNK_FRAMES;
        mm[i] = MelClip{clips[i].pcm, (long long)pl.n, (long long)chunk * CHUNK_FRAMES, (int)fb, (int)pl.f_end,
                        own && whole ? i : -1, 0};
        if (own && !whole) {
            mx[n_max_pass++] = MelClip{clips[i].pcm, (long long)pl.n, 0, 0, (int)pl.F, i, 0};
            max_pass_frames += pl.F;
        }
        range_frames += pl.f_end - fb;
        int64_t tok = pl.tok0;
        for (int64_t c = pl.c_first; c < pl.c_last; c++, chunk++) {
            const int nf = (int)std::min<int64_t>(CHUNK_FRAMES, pl.F - c * CHUNK_FRAMES);
            const int nt = (int)chunk_tokens(nf);
            // the chunk's tokens need conv3 rows t < nt, conv2 rows t < 2 nt and
            // conv1 rows t < 4 nt (kernel 3, stride 2, padding 1)
            sc[chunk] = StemChunk{i, (int)(chunk * CHUNK_FRAMES), nf, std::min(400, 4 * nt)};
            ct[chunk] = make_int2((int)tok, nt);
            tok += nt;
        }
    }
    // conv2 / conv3 tile lists per stem group (chunk index within the group)
    int *t2 = reinterpret_cast<int *>(H + tl.tiles2);
    int *t3 = reinterpret_cast<int *>(H + tl.tiles3);
    std::vector<int> g_off2, g_n2, g_off3, g_n3;
    {
        int o2 = 0, o3 = 0;
        for (int64_t g0 = 0; g0 < n_chunks; g0 += h->stem_group) {
            const int gc = (int)std::min<int64_t>(h->stem_group, n_chunks - g0);
            g_off2.push_back(o2);
            g_off3.push_back(o3);
            for (int j = 0; j < gc; j++) {
                const int nt = ct[g0 + j].y;
                const int n2 = (std::min(200, 2 * nt) + 3) / 4, n3 = (nt + 7) / 8;
                for (int m = 0; m < n2; m++) t2[o2++] = j * 256 + m;
                for (int m = 0; m < n3; m++) t3[o3++] = j * 256 + m;
            }
            // CTA pairs take two list entries at a time: pad to an even count
            if ((o2 - g_off2.back()) & 1) t2[o2++] = -1;
            if ((o3 - g_off3.back()) & 1) t3[o3++] = -1;
            g_n2.push_back(o2 - g_off2.back());
            g_n3.push_back(o3 - g_off3.back());
        }
    }
    FwdPlan P;
    P.n_clips = n_clips;
    P.n_chunks = n_chunks;
    P.T = T;
    P.n_max_pass = n_max_pass;
    P.max_clip_frames = max_clip_frames;
    P.max_range_frames = max_range_frames;
    P.max_pass_frames = max_pass_frames;
    P.range_frames = range_frames;
    P.sc = sc;
    P.ct = ct;
    P.g_off2 = std::move(g_off2);
    P.g_n2 = std::move(g_n2);
    P.g_off3 = std::move(g_off3);
    P.g_n3 = std::move(g_n3);

    // Whole forwards run as one CUDA graph once a request shape repeats: the
    // second consecutive call of one shape (clip and chunk structure, taps)
    // captures it, later calls of that shape replay it with their own tables
    // (copied, in stream order, into the tables the graph reads).  The graph
    // writes the rows to the workspace's output area, and one device copy
    // moves them to the caller's buffer, so pieces of a long clip with
    // different output ranges share the graph.  A request of a new shape runs
    // launch by launch and never pays for a capture.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    CUDA_TRY(h, cudaStreamIsCapturing(h->stream, &cs));
    const int n_taps = (int)h->tap_layers.size();
    const bool graphable = stage == MOSS_ENC_STAGE_ADAPTER && !h->profiling && h->stream != nullptr &&
                           cs == cudaStreamCaptureStatusNone;
    const size_t out_bytes = (size_t)T * DOUT * (h->cfg.out_dtype == MOSS_ENC_OUT_F32 ? 4 : 2);
    auto rows_to_caller = [&]() -> moss_enc_status {
        if (out != h->out_stage)
            CUDA_TRY(h, cudaMemcpyAsync(out, h->out_stage, out_bytes, cudaMemcpyDeviceToDevice, h->stream));
        return MOSS_ENC_OK;
    };
    std::vector<uint8_t> key;
    if (graphable) key = shape_key(P, tap_out, n_taps);
    if (graphable && h->graph_exec && h->graph_key == key) {
        TRY(tab_upload(h, h->d_tab_graph));
        h->launches += h->graph_launches;
        CUDA_TRY(h, cudaGraphLaunch(h->graph_exec, h->stream));
        return rows_to_caller();
    }
    if (!graphable || key != h->last_key) {
        if (graphable) h->last_key = std::move(key);
        TRY(tab_upload(h));
        return forward_launch(h, P, static_cast<uint8_t *>(h->d_tab), stage, out, tap_out);
    }
    if (h->graph_exec) {
        cudaGraphExecDestroy(h->graph_exec);
        h->graph_exec = nullptr;
    }
    TRY(tab_upload(h, h->d_tab_graph));
    const int64_t launches0 = h->launches;
    CUDA_TRY(h, cudaStreamBeginCapture(h->stream, cudaStreamCaptureModeThreadLocal));
    const moss_enc_status st = forward_launch(h, P, static_cast<uint8_t *>(h->d_tab_graph), stage, h->out_stage, tap_out);
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(h->stream, &g);
    if (st != MOSS_ENC_OK || ce != cudaSuccess) {
        if (g) cudaGraphDestroy(g);
        cudaGetLastError();
        return st != MOSS_ENC_OK ? st : fail(h, MOSS_ENC_ERR_CUDA, std::string("graph capture: ") + cudaGetErrorString(ce));
    }
    const cudaError_t ie = cudaGraphInstantiate(&h->graph_exec, g, 0);
    cudaGraphDestroy(g);
    if (ie != cudaSuccess) {
        h->graph_exec = nullptr;
        return fail(h, MOSS_ENC_ERR_CUDA, std::string("graph instantiate: ") + cudaGetErrorString(ie));
    }
    h->graph_key = std::move(key);
    h->graph_launches = h->launches - launches0;
    CUDA_TRY(h, cudaGraphLaunch(h->graph_exec, h->stream));
    return rows_to_caller();
}


extern "C" moss_enc_status moss_enc_forward(moss_enc *h, const moss_enc_clip *clips, int n_clips, void *rows_out,
                                            int64_t *row_offsets)
{
    return forward_impl(h, clips, n_clips, MOSS_ENC_STAGE_ADAPTER, rows_out, row_offsets);
}

extern "C" moss_enc_status moss_enc_forward_stage(moss_enc *h, const moss_enc_clip *clips, int n_clips, int stage,
                                                  void *out, int64_t *row_offsets)
{
    return forward_impl(h, clips, n_clips, stage, out, row_offsets);
}

extern "C" int64_t moss_enc_tap_weight_count(void) { return head_count(); }

extern "C" moss_enc_status moss_enc_set_taps(moss_enc *h, const int *layers, int n_taps, const void *weights,
                                             size_t bytes, int weights_on_device)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (n_taps < 0 || n_taps > MOSS_ENC_MAX_TAPS || (n_taps > 0 && !layers))
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad tap list");
    for (int t = 0; t < n_taps; t++)
        if (layers[t] < 0 || layers[t] >= h->cfg.n_layers) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "tap layer out of range");
    if (weights && (int64_t)bytes != 2 * head_count() * n_taps)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "tap weight blob has the wrong size");
    // pending work may still read the old tap weights
    CUDA_TRY(h, cudaStreamSynchronize(h->stream));
    if (h->graph_exec) {
        cudaGraphExecDestroy(h->graph_exec);
        h->graph_exec = nullptr;
        h->graph_key.clear();
        h->last_key.clear();
    }
    if (h->tap_wmem) {
        cudaFree(h->tap_wmem);
        h->tap_wmem = nullptr;
    }
    h->tap_layers.clear();
    h->tap_heads.clear();
    if (n_taps == 0) return MOSS_ENC_OK;
    std::vector<HeadDev> heads(n_taps, h->head);
    if (weights) {
        size_t off = 0;
        auto take = [&](size_t b) {
            size_t r = off;
            off += (b + 255) & ~size_t(255);
            return r;
        };
        std::vector<HeadOff> o(n_taps);
        for (int t = 0; t < n_taps; t++) o[t] = head_take(take, take);
        std::vector<uint16_t> host;
        const uint16_t *p = static_cast<const uint16_t *>(weights);
        if (weights_on_device) {
            host.resize((size_t)head_count() * n_taps);
            CUDA_TRY(h, cudaMemcpy(host.data(), weights, bytes, cudaMemcpyDeviceToHost));
            p = host.data();
        }
        std::vector<uint8_t> pk(off, 0);
        for (int t = 0; t < n_taps; t++) p = head_pack(o[t], pk.data(), p);
        if (cudaMalloc(&h->tap_wmem, off) != cudaSuccess) {
            h->tap_wmem = nullptr;
            return fail(h, MOSS_ENC_ERR_OOM, "tap weights");
        }
        CUDA_TRY(h, cudaMemcpy(h->tap_wmem, pk.data(), off, cudaMemcpyHostToDevice));
        for (int t = 0; t < n_taps; t++) heads[t] = head_bind(o[t], static_cast<uint8_t *>(h->tap_wmem));
    }
    h->tap_layers.assign(layers, layers + n_taps);
    h->tap_heads = std::move(heads);
    return MOSS_ENC_OK;
}

extern "C" moss_enc_status moss_enc_forward_taps(moss_enc *h, const moss_enc_clip *clips, int n_clips, void *rows_out,
                                                 void *const *tap_rows, int64_t *row_offsets)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (!h->tap_layers.empty() && !tap_rows) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "null tap_rows");
    return forward_impl(h, clips, n_clips, MOSS_ENC_STAGE_ADAPTER, rows_out, row_offsets,
                        h->tap_layers.empty() ? nullptr : tap_rows);
}

extern "C" moss_enc_status moss_enc_forward_host(moss_enc *h, const float *const *pcm_host, const int64_t *n_samples,
                                                 int n_clips, void *rows_host, int64_t *row_offsets)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (n_clips < 0 || n_clips > h->cfg.max_clips || (n_clips > 0 && (!pcm_host || !n_samples)) || !row_offsets)
        return fail(h, n_clips > h->cfg.max_clips ? MOSS_ENC_ERR_CAPACITY : MOSS_ENC_ERR_INVALID_ARG, "bad argument");
    int64_t total = 0;
    for (int i = 0; i < n_clips; i++) {
        if (n_samples[i] < 0 || (n_samples[i] > 0 && !pcm_host[i])) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad clip");
        total += (n_samples[i] + 3) & ~int64_t(3);  // keep every clip 16-byte aligned
    }
    if (total > h->cfg.max_samples) return fail(h, MOSS_ENC_ERR_CAPACITY, "clips exceed max_samples");
    std::vector<moss_enc_clip> cl(n_clips);
    int64_t o = 0;
    for (int i = 0; i < n_clips; i++) {
        if (n_samples[i] > 0)
            CUDA_TRY(h, cudaMemcpyAsync(h->pcm_stage + o, pcm_host[i], sizeof(float) * n_samples[i],
                                        cudaMemcpyHostToDevice, h->stream));
        cl[i] = moss_enc_clip{h->pcm_stage + o, n_samples[i], 0, n_samples[i], nullptr};
        o += (n_samples[i] + 3) & ~int64_t(3);
    }
    TRY(forward_impl(h, cl.data(), n_clips, MOSS_ENC_STAGE_ADAPTER, h->out_stage, row_offsets));
    const int64_t T = row_offsets[n_clips];
    const size_t esz = h->cfg.out_dtype == MOSS_ENC_OUT_F32 ? 4 : 2;
    if (T > 0) {
        if (!rows_host) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "null rows_host");
        CUDA_TRY(h, cudaMemcpyAsync(rows_host, h->out_stage, esz * T * DOUT, cudaMemcpyDeviceToHost, h->stream));
    }
    return moss_enc_synchronize(h);
}

// ------------------------------------------------------------- measurement

extern "C" moss_enc_status moss_enc_profile_enable(moss_enc *h, int max_launches)
{
    if (!h || max_launches < 0) return MOSS_ENC_ERR_INVALID_ARG;
    CUDA_TRY(h, cudaStreamSynchronize(h->stream));
    for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
    h->prof_ev.clear();
    h->prof_rec.clear();
    h->profiling = max_launches > 0;
    for (int i = 0; i < 2 * max_launches; i++) {
        cudaEvent_t e;
        CUDA_TRY(h, cudaEventCreate(&e));
        h->prof_ev.push_back(e);
    }
    h->prof_rec.reserve(max_launches);
    return MOSS_ENC_OK;
}

extern "C" int moss_enc_profile_read(moss_enc *h, moss_enc_kernel_stat *out, int max)
{
    if (!h || (max > 0 && !out)) return -1;
    if (cudaStreamSynchronize(h->stream) != cudaSuccess) return -1;
    std::vector<moss_enc_kernel_stat> agg;
    for (const auto &r : h->prof_rec) {
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, h->prof_ev[r.e0], h->prof_ev[r.e0 + 1]) != cudaSuccess) return -1;
        moss_enc_kernel_stat *st = nullptr;
        for (auto &a : agg)
            if (std::strncmp(a.name, r.name, sizeof(a.name)) == 0) st = &a;
        if (!st) {
            agg.push_back(moss_enc_kernel_stat{});
            st = &agg.back();
            std::strncpy(st->name, r.name, sizeof(st->name) - 1);
        }
        st->launches++;
        st->ms += ms;
        st->flops += r.flops;
        st->bytes += r.bytes;
    }
    h->prof_rec.clear();
    const int n = (int)std::min<size_t>(agg.size(), (size_t)std::max(max, 0));
    for (int i = 0; i < n; i++) out[i] = agg[i];
    return n;
}

extern "C" int64_t moss_enc_launch_count(const moss_enc *h) { return h ? h->launches : -1; }

// --------------------------------------------------------------- one GEMM

template <int BN>
static moss_enc_status gemm_one(moss_enc *h, const bf16 *A, const bf16 *B, const float *bias, void *out, int M,
                                int N, int K, int epi, int pair)
{
    GemmArgs a{};
    a.bias = bias;
    a.out = out;
    a.ldo = N;
    switch (epi * 2 + (pair ? 1 : 0)) {
    case EPI_BF16 * 2: return gemm<BN, EPI_BF16>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_GELU_BF16 * 2: return gemm<BN, EPI_GELU_BF16>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_RESID_F32 * 2: return gemm<BN, EPI_RESID_F32>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_F32 * 2: return gemm<BN, EPI_F32>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_BF16 * 2 + 1: return gemm2<BN, EPI_BF16>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_GELU_BF16 * 2 + 1: return gemm2<BN, EPI_GELU_BF16>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_RESID_F32 * 2 + 1: return gemm2<BN, EPI_RESID_F32>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_F32 * 2 + 1: return gemm2<BN, EPI_F32>(h, "gemm_api", A, M, K, B, N, a);
    default: return fail(h, MOSS_ENC_ERR_INVALID_ARG, "unsupported epilogue");
    }
}

template <int BN>
static cudaError_t gemm_api_attrs()
{
    cudaError_t e;
    if ((e = gemm_attr<BN, EPI_BF16>()) != cudaSuccess) return e;
    if ((e = gemm_attr<BN, EPI_GELU_BF16>()) != cudaSuccess) return e;
    if ((e = gemm_attr<BN, EPI_RESID_F32>()) != cudaSuccess) return e;
    if ((e = gemm_attr<BN, EPI_F32>()) != cudaSuccess) return e;
    if ((e = gemm2_attr<BN, EPI_BF16>()) != cudaSuccess) return e;
    if ((e = gemm2_attr<BN, EPI_GELU_BF16>()) != cudaSuccess) return e;
    if ((e = gemm2_attr<BN, EPI_RESID_F32>()) != cudaSuccess) return e;
    return gemm2_attr<BN, EPI_F32>();
}

extern "C" moss_enc_status moss_enc_gemm(moss_enc *h, const void *A, const void *B, const float *bias, void *out,
                                         int M, int N, int K, int epilogue, int block_n, int cta_pair)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (!A || !B || !bias || !out || M < 0 || N <= 0 || K <= 0 || K % 64 != 0)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad gemm arguments");
    if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(bias)) & 15)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "A, B and bias must be 16-byte aligned");
    static bool attrs_done = false;
    if (!attrs_done) {
        CUDA_TRY(h, gemm_api_attrs<128>());
        CUDA_TRY(h, gemm_api_attrs<160>());
        CUDA_TRY(h, gemm_api_attrs<192>());
        CUDA_TRY(h, gemm_api_attrs<256>());
        CUDA_TRY(h, (gemm2_attr<320, EPI_BF16>()));
        CUDA_TRY(h, (gemm2_attr<320, EPI_GELU_BF16>()));
        CUDA_TRY(h, (gemm2_attr<320, EPI_RESID_F32>()));
        CUDA_TRY(h, (gemm2_attr<320, EPI_F32>()));
        attrs_done = true;
    }
    const bf16 *a = static_cast<const bf16 *>(A), *b = static_cast<const bf16 *>(B);
    if (N % block_n != 0) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "N % block_n != 0");
    switch (block_n) {
    case 128: return gemm_one<128>(h, a, b, bias, out, M, N, K, epilogue, cta_pair);
    case 160: return gemm_one<160>(h, a, b, bias, out, M, N, K, epilogue, cta_pair);
    case 192: return gemm_one<192>(h, a, b, bias, out, M, N, K, epilogue, cta_pair);
    case 256: return gemm_one<256>(h, a, b, bias, out, M, N, K, epilogue, cta_pair);
    case 320: {
        if (!cta_pair) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "block_n 320 needs cta_pair");
        GemmArgs g{};
        g.bias = bias;
        g.out = out;
        g.ldo = N;
        switch (epilogue) {
        case EPI_BF16: return gemm2<320, EPI_BF16>(h, "gemm_api", a, M, K, b, N, g);
        case EPI_GELU_BF16: return gemm2<320, EPI_GELU_BF16>(h, "gemm_api", a, M, K, b, N, g);
        case EPI_RESID_F32: return gemm2<320, EPI_RESID_F32>(h, "gemm_api", a, M, K, b, N, g);
        case EPI_F32: return gemm2<320, EPI_F32>(h, "gemm_api", a, M, K, b, N, g);
        default: return fail(h, MOSS_ENC_ERR_INVALID_ARG, "unsupported epilogue");
        }
    }
    default: return fail(h, MOSS_ENC_ERR_INVALID_ARG, "block_n must be 128, 160, 192, 256 or 320");
    }
}

template <int BN>
static moss_enc_status gemm_q4_one(moss_enc *h, const bf16 *A, const QW &B, const float *bias, void *out, int M,
                                   int N, int K, int epi)
{
    GemmArgs a{};
    a.bias = bias;
    a.out = out;
    a.ldo = N;
    switch (epi) {
    case EPI_BF16: return gemm2q<BN, EPI_BF16>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_GELU_BF16: return gemm2q<BN, EPI_GELU_BF16>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_RESID_F32: return gemm2q<BN, EPI_RESID_F32>(h, "gemm_api", A, M, K, B, N, a);
    case EPI_F32: return gemm2q<BN, EPI_F32>(h, "gemm_api", A, M, K, B, N, a);
    default: return fail(h, MOSS_ENC_ERR_INVALID_ARG, "unsupported epilogue");
    }
}

template <int BN>
static cudaError_t gemm_q4_api_attrs()
{
    cudaError_t e;
    if ((e = gemm2q_attr<BN, EPI_BF16>()) != cudaSuccess) return e;
    if ((e = gemm2q_attr<BN, EPI_GELU_BF16>()) != cudaSuccess) return e;
    if ((e = gemm2q_attr<BN, EPI_RESID_F32>()) != cudaSuccess) return e;
    return gemm2q_attr<BN, EPI_F32>();
}

extern "C" moss_enc_status moss_enc_gemm_q4(moss_enc *h, const void *A, const void *Bq, const float *Bs,
                                            const float *bias, void *out, int M, int N, int K, int epilogue,
                                            int block_n)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (!A || !Bq || !Bs || !bias || !out || M < 0 || N <= 0 || K <= 0 || K % 128 != 0)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad gemm arguments");
    if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(Bq) | reinterpret_cast<uintptr_t>(Bs) |
         reinterpret_cast<uintptr_t>(bias)) & 15)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "A, Bq, Bs and bias must be 16-byte aligned");
    if (N % block_n != 0 || N % 4 != 0) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "N % block_n != 0");
    static bool attrs_done = false;
    if (!attrs_done) {
        CUDA_TRY(h, gemm_q4_api_attrs<128>());
        CUDA_TRY(h, gemm_q4_api_attrs<160>());
        CUDA_TRY(h, gemm_q4_api_attrs<256>());
        CUDA_TRY(h, gemm_q4_api_attrs<320>());
        attrs_done = true;
    }
    QW q;
    q.codes = static_cast<const uint8_t *>(Bq);
    q.scales = Bs;
    q.kq = K;
    const bf16 *a = static_cast<const bf16 *>(A);
    switch (block_n) {
    case 128: return gemm_q4_one<128>(h, a, q, bias, out, M, N, K, epilogue);
    case 160: return gemm_q4_one<160>(h, a, q, bias, out, M, N, K, epilogue);
    case 256: return gemm_q4_one<256>(h, a, q, bias, out, M, N, K, epilogue);
    case 320: return gemm_q4_one<320>(h, a, q, bias, out, M, N, K, epilogue);
    default: return fail(h, MOSS_ENC_ERR_INVALID_ARG, "block_n must be 128, 160, 256 or 320");
    }
}

extern "C" moss_enc_status moss_enc_gemm_f8(moss_enc *h, const void *A8, const void *B8, const float *sa,
                                            const float *sb, const float *bias, void *out, int M, int N, int K,
                                            int epilogue, int block_n)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (!A8 || !B8 || !sa || !sb || !bias || !out || M < 0 || N <= 0 || K <= 0 || K % 256 != 0)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad gemm arguments");
    if ((reinterpret_cast<uintptr_t>(A8) | reinterpret_cast<uintptr_t>(B8) | reinterpret_cast<uintptr_t>(bias) |
         reinterpret_cast<uintptr_t>(sb)) & 15)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "A8, B8, sb and bias must be 16-byte aligned");
    if (block_n != 128 && block_n != 256) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "block_n must be 128 or 256");
    if (N % block_n != 0) return fail(h, MOSS_ENC_ERR_INVALID_ARG, "N % block_n != 0");
    GemmArgs a{};
    a.bias = bias;
    a.out = out;
    a.ldo = N;
    a.row_scale = sa;
    a.col_scale = sb;
    const uint8_t *a8 = static_cast<const uint8_t *>(A8), *b8 = static_cast<const uint8_t *>(B8);
    switch (epilogue * 2 + (block_n == 256 ? 1 : 0)) {
    case EPI_BF16 * 2: return gemm2f8<128, EPI_BF16>(h, "gemm_api", a8, M, K, b8, N, a);
    case EPI_BF16 * 2 + 1: return gemm2f8<256, EPI_BF16>(h, "gemm_api", a8, M, K, b8, N, a);
    case EPI_GELU_BF16 * 2: return gemm2f8<128, EPI_GELU_BF16>(h, "gemm_api", a8, M, K, b8, N, a);
    case EPI_GELU_BF16 * 2 + 1: return gemm2f8<256, EPI_GELU_BF16>(h, "gemm_api", a8, M, K, b8, N, a);
    default: return fail(h, MOSS_ENC_ERR_INVALID_ARG, "epilogue must be 0 or 1");
    }
}

extern "C" moss_enc_status moss_enc_gemm_nvf4(moss_enc *h, const void *A4, const void *sfa, const float *ga,
                                              const void *B4, const void *sfb, const float *gb, const float *bias,
                                              void *out, int M, int N, int K, int epilogue)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (!A4 || !sfa || !ga || !B4 || !sfb || !gb || !bias || !out || M < 0 || N <= 0 || K <= 0 || K % 256 != 0 ||
        N % 128 != 0)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad gemm arguments");
    if ((reinterpret_cast<uintptr_t>(A4) | reinterpret_cast<uintptr_t>(B4) | reinterpret_cast<uintptr_t>(sfa) |
         reinterpret_cast<uintptr_t>(sfb) | reinterpret_cast<uintptr_t>(gb) | reinterpret_cast<uintptr_t>(bias)) & 15)
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "A4, B4, the scale atoms, gb and bias must be 16-byte aligned");
    GemmArgs a{};
    a.bias = bias;
    a.out = out;
    a.ldo = N;
    a.row_scale = ga;
    a.col_scale = gb;
    a.sfa = static_cast<const uint8_t *>(sfa);
    a.sfb = static_cast<const uint8_t *>(sfb);
    const uint8_t *a4 = static_cast<const uint8_t *>(A4), *b4 = static_cast<const uint8_t *>(B4);
    switch (epilogue) {
    case EPI_BF16: return gemm_nvf4<EPI_BF16>(h, "gemm_api", a4, M, K, b4, N, a);
    case EPI_GELU_BF16: return gemm_nvf4<EPI_GELU_BF16>(h, "gemm_api", a4, M, K, b4, N, a);
    default: return fail(h, MOSS_ENC_ERR_INVALID_ARG, "epilogue must be 0 or 1");
    }
}

extern "C" moss_enc_status moss_enc_nvf4_quant_weights(const void *w, int n, int k, int parts, void *codes, void *sfa,
                                                       float *g)
{
    if (!w || !codes || !sfa || !g || n <= 0 || k <= 0 || parts <= 0 || n % parts != 0 || (n / parts) % 128 != 0 ||
        k % 64 != 0)
        return MOSS_ENC_ERR_INVALID_ARG;
    quantise_nvfp4_to(static_cast<const uint16_t *>(w), n, k, parts, static_cast<uint8_t *>(codes),
                      static_cast<uint8_t *>(sfa), g);
    return MOSS_ENC_OK;
}

extern "C" moss_enc_status moss_enc_nvf4_quant_rows(moss_enc *h, const float *x, void *codes, void *sfa, float *g,
                                                    int M)
{
    if (!h) return MOSS_ENC_ERR_INVALID_ARG;
    if (M < 0 || (M > 0 && (!x || !codes || !sfa || !g)))
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "bad quantisation arguments");
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(codes) & 1))
        return fail(h, MOSS_ENC_ERR_INVALID_ARG, "x must be 16-byte and codes 2-byte aligned");
    if (M == 0) return MOSS_ENC_OK;
    CUDA_TRY(h, launch_k(h, nvf4_rows1280_kernel<false>, dim3((M + 7) / 8), dim3(256), 0, x, (const float *)nullptr,
                         (const float *)nullptr, static_cast<uint8_t *>(codes), static_cast<uint8_t *>(sfa), g, M));
    return MOSS_ENC_OK;
}

// --------------------------------------------------------- GELU self-test

__global__ void gelu_check_kernel(float lo, float hi, int n, unsigned int *max_err_bits)
{
    float worst = 0.0f;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float x = lo + (hi - lo) * ((float)i / (float)(n - 1));
        const float ref = gelu_erf(x);
        const float2 g2 = gelu2(make_float2(x, -x));
        const float d = fmaxf(fabsf(gelu_fast(x) - ref), fmaxf(fabsf(g2.x - ref), fabsf(g2.y - gelu_erf(-x))));
        worst = fmaxf(worst, d / fmaxf(1.0f, fabsf(x)));
    }
    atomicMax(max_err_bits, __float_as_uint(worst));  // non-negative floats order like their bits
}

extern "C" moss_enc_status moss_enc_selftest_gelu(moss_enc *h, float *max_rel_err)
{
    if (!h || !max_rel_err) return MOSS_ENC_ERR_INVALID_ARG;
    unsigned int *d = reinterpret_cast<unsigned int *>(h->err) + 8;  // spare words of the flag block
    CUDA_TRY(h, cudaMemsetAsync(d, 0, sizeof(unsigned int), h->stream));
    gelu_check_kernel<<<h->num_sms, 256, 0, h->stream>>>(-12.0f, 12.0f, 1 << 22, d);
    CUDA_TRY(h, cudaGetLastError());
    unsigned int bits = 0;
    CUDA_TRY(h, cudaMemcpyAsync(&bits, d, sizeof(bits), cudaMemcpyDeviceToHost, h->stream));
    CUDA_TRY(h, cudaStreamSynchronize(h->stream));
    std::memcpy(max_rel_err, &bits, sizeof(float));
    return MOSS_ENC_OK;
}

// ------------------------------------------------ bounded-wait self-test

// One thread waits on an mbarrier that nothing arrives at, with the given
// limit, the way every pipeline wait in the kernels is bounded.  The wait
// gives up, raises the timeout bit of the handle's device flag, and returns.
__global__ void wait_timeout_check_kernel(int *err, unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar, 0)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(err, DEV_ERR_TIMEOUT);
            return;
        }
    }
}

extern "C" moss_enc_status moss_enc_selftest_timeout(moss_enc *h, int limit_ms)
{
    if (!h || limit_ms < 1 || limit_ms > 2000) return MOSS_ENC_ERR_INVALID_ARG;
    wait_timeout_check_kernel<<<1, 32, 0, h->stream>>>(h->err, (unsigned long long)limit_ms * 1000000ull);
    CUDA_TRY(h, cudaGetLastError());
    return MOSS_ENC_OK;
}

// ------------------------------------------------- allocation-free log-mel
//
// Scratch for moss_enc_logmel_static: a fixed-size device array, laid out as
// [log-mel kernel tables (Mel4Tab) | main-pass MelClip x 64 | max-pass
// MelClip x 64 | log_max
// source pointers x 64 | ordered-int maxima x 64].  Nothing here allocates.

namespace {
constexpr int STATIC_MAX_CLIPS = MOSS_ENC_STATIC_MAX_CLIPS;
constexpr size_t ST_TABLES = 0;
constexpr size_t ST_MAIN = (sizeof(Mel4Tab) + 255) & ~size_t(255);
constexpr size_t ST_MAXP = ST_MAIN + ((sizeof(MelClip) * STATIC_MAX_CLIPS + 255) & ~size_t(255));
constexpr size_t ST_SRC = ST_MAXP + ((sizeof(MelClip) * STATIC_MAX_CLIPS + 255) & ~size_t(255));
constexpr size_t ST_GMAX = ST_SRC + ((sizeof(float *) * STATIC_MAX_CLIPS + 255) & ~size_t(255));
constexpr size_t ST_USED = ST_GMAX + sizeof(int) * STATIC_MAX_CLIPS;
constexpr size_t ST_BYTES = 24576;
static_assert(ST_USED <= ST_BYTES, "static log-mel scratch too small");

// Per-call descriptors staged on the host before one copy into the array.
struct StaticStage {
    MelClip main[STATIC_MAX_CLIPS];
    MelClip maxp[STATIC_MAX_CLIPS];
    const float *src[STATIC_MAX_CLIPS];
};

constexpr int STATIC_MAX_DEVICES = 64;
std::mutex g_static_mu;
uint8_t *g_static_ptr[STATIC_MAX_DEVICES] = {};
int g_static_sms[STATIC_MAX_DEVICES] = {};
}  // namespace

static __device__ __align__(256) uint8_t g_logmel_scratch[ST_BYTES];

// Device address of the scratch on the current device; the first call per
// device looks it up and writes the constant tables into it.
static moss_enc_status static_scratch(uint8_t **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= STATIC_MAX_DEVICES) return MOSS_ENC_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_logmel_scratch) != cudaSuccess || !p) return MOSS_ENC_ERR_CUDA;
        if (cudaFuncSetAttribute(logmel4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Mel4Smem)) !=
                cudaSuccess ||
            cudaFuncSetAttribute(logmel4_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
            return MOSS_ENC_ERR_CUDA;
        MelTables tab;
        static Mel4Tab tab4;  // built once under the lock (too large for the stack)
        if (!build_mel_tables(&tab) || !build_mel4_tab(tab, &tab4)) return MOSS_ENC_ERR_INVALID_ARG;
        if (cudaMemcpy(static_cast<uint8_t *>(p) + ST_TABLES, &tab4, sizeof(tab4), cudaMemcpyHostToDevice) != cudaSuccess)
            return MOSS_ENC_ERR_CUDA;
        if (cudaDeviceGetAttribute(&g_static_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOSS_ENC_ERR_CUDA;
        g_static_ptr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_static_ptr[dev];
    return MOSS_ENC_OK;
}

extern "C" moss_enc_status moss_enc_logmel_static(const moss_enc_clip *clips, int n_clips, float *const *mel_out,
                                                  float *log_max_out, void *stream)
{
    if (n_clips < 0 || (n_clips > 0 && (!clips || !mel_out))) return MOSS_ENC_ERR_INVALID_ARG;
    if (n_clips > STATIC_MAX_CLIPS) return MOSS_ENC_ERR_CAPACITY;
    if (n_clips == 0) return MOSS_ENC_OK;
    cudaStream_t st = (cudaStream_t)stream;
    StaticStage stage;
    std::memset(&stage, 0, sizeof(stage));
    int n_max = 0;
    int64_t max_clip = 0;
    for (int i = 0; i < n_clips; i++) {
        const moss_enc_clip &c = clips[i];
        // a clip with samples is read by the maximum pass even when its range is empty
        if (c.n_samples > 0 && !c.pcm) return MOSS_ENC_ERR_INVALID_ARG;
        ClipPlan pl;
        if (!plan_clip(c.n_samples, c.begin, c.end, &pl) || pl.F > INT32_MAX) return MOSS_ENC_ERR_INVALID_ARG;
        const int64_t nf = pl.f_end - pl.f_begin;
        if (nf > 0 && !mel_out[i]) return MOSS_ENC_ERR_INVALID_ARG;
        const bool whole = pl.f_begin == 0 && pl.f_end == pl.F;
        const bool own = c.log_max == nullptr;
        stage.src[i] = c.log_max;
        // every clip has its own output buffer, so each clip gets its own
        // launch below and writes from row 0 of that buffer
        stage.main[i] = MelClip{c.pcm, (long long)pl.n, 0, (int)pl.f_begin, (int)pl.f_end, own && whole ? i : -1, 0};
        if (own && !whole) stage.maxp[n_max++] = MelClip{c.pcm, (long long)pl.n, 0, 0, (int)pl.F, i, 0};
        max_clip = std::max(max_clip, pl.F);
    }
    // The descriptors are copied from this call's stack frame: a captured copy
    // would be replayed after the frame is gone, so a capturing stream is refused.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return MOSS_ENC_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return MOSS_ENC_ERR_INVALID_ARG;
    uint8_t *S = nullptr;
    moss_enc_status s = static_scratch(&S);
    if (s != MOSS_ENC_OK) return s;
    MelClip *d_main = reinterpret_cast<MelClip *>(S + ST_MAIN);
    MelClip *d_maxp = reinterpret_cast<MelClip *>(S + ST_MAXP);
    const float *const *d_src = reinterpret_cast<const float *const *>(S + ST_SRC);
    int *d_gmax = reinterpret_cast<int *>(S + ST_GMAX);
    const Mel4Tab *d_tab = reinterpret_cast<const Mel4Tab *>(S + ST_TABLES);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOSS_ENC_ERR_CUDA;
    const int64_t max_grid = 4 * (int64_t)g_static_sms[dev];
    auto grid_for = [&](int64_t blocks) { return (int)std::max<int64_t>(1, std::min<int64_t>(blocks, max_grid)); };
    if (cudaMemcpyAsync(S + ST_MAIN, stage.main, sizeof(stage.main), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(S + ST_MAXP, stage.maxp, sizeof(stage.maxp), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(S + ST_SRC, stage.src, sizeof(stage.src), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOSS_ENC_ERR_CUDA;
    // the maxima start at -inf or at the caller's value
    gmax_init_kernel<<<1, STATIC_MAX_CLIPS, 0, st>>>(d_gmax, d_src, n_clips);
    if (n_max > 0)
        logmel4_kernel<<<grid_for(n_max * ((max_clip + MEL4_FRAMES - 1) / MEL4_FRAMES)), MEL4_THREADS, sizeof(Mel4Smem),
                         st>>>(d_maxp, n_max, d_tab, nullptr, d_gmax, 0);
    for (int i = 0; i < n_clips; i++) {
        const int nf = stage.main[i].f_end - stage.main[i].f_begin;
        if (nf <= 0) continue;
        logmel4_kernel<<<grid_for((nf + MEL4_FRAMES - 1) / MEL4_FRAMES), MEL4_THREADS, sizeof(Mel4Smem), st>>>(
            d_main + i, 1, d_tab, mel_out[i], d_gmax, 1);
    }
    for (int i = 0; i < n_clips; i++) {
        const int64_t nf = stage.main[i].f_end - stage.main[i].f_begin;
        if (nf > 0)
            mel_normalize_kernel<<<(int)std::min<int64_t>(4096, (nf * 128 + 255) / 256), 256, 0, st>>>(mel_out[i], nf * 128, d_gmax + i);
        if (log_max_out) gmax_export_kernel<<<1, 32, 0, st>>>(d_gmax + i, log_max_out + i);
    }
    return cudaGetLastError() == cudaSuccess ? MOSS_ENC_OK : MOSS_ENC_ERR_CUDA;
}
