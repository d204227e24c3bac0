// Whisper-style log-mel front end (fp32, CUDA cores).
//
// Blocks of 16 consecutive frames of a clip: the PCM span those frames cover
// (160*15 + 400 samples) is copied once into shared memory, with reflect
// padding applied only at the true clip ends.  Frames are transformed two at
// a time: frame a as the real part and frame b as the imaginary part of one
// 400-point complex DFT, computed as 20 x 20 (two passes of 20-point DFTs,
// each a 4-point and a 5-point stage, with the 400-point twiddles between the
// passes).  The two real spectra are separated with X_a[k] = (Z[k] + conj
// Z[-k]) / 2, X_b[k] = (Z[k] - conj Z[-k]) / 2i, squared, pushed through the
// banded mel filterbank, and log10'd.  A block's maximum goes to the clip's
// maximum with one ordered-integer atomicMax.
#pragma once

#include "common.cuh"

namespace moss {

static constexpr int MEL_BAND = 16;  // max nonzero FFT bins of one mel filter

// One clip's frame range for a log-mel launch: frames [f_begin, f_end), frame
// f to output row out_row0 + (f - f_begin).  gslot >= 0 names the per-clip
// maximum this range folds into (atomicMax); -1 folds into nothing.
struct MelClip {
    const float *pcm;
    long long n;
    long long out_row0;
    int f_begin, f_end;
    int gslot;
    int pad;
};

// The transform and filterbank in their plain form (built on the host from
// the definitions; the kernel's tables, Mel4Tab, are derived from them).
struct MelTables {
    float2 tw400[400];            // exp(-2 pi i k / 400)
    float hann[400];              // periodic Hann
    int band_lo[128];             // first nonzero bin of each filter
    float band_w[128][MEL_BAND];  // filter weights on bins band_lo .. band_lo+15
    int band_n[128];              // nonzero bins of each filter (<= MEL_BAND)
};

__device__ __forceinline__ float2 cmul(float2 a, float2 b)
{
    return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

// 20-point DFT in registers: X[k] = sum_n x[n] exp(-2 pi i n k / 20).
// n = nb + 5 na, k = 4 kb + ka:  4-point DFTs over na, twiddle
// exp(-2 pi i nb ka / 20) (compile-time constants), then 5-point DFTs over nb.
// Each complex value's real and imaginary parts sit in the two lanes of the
// paired fp32 instructions: the 4- and 5-point stages' additions and
// real-constant products take one paired instruction per complex value;
// (-i) z is the lane swap (z.y, -z.x).
__device__ __forceinline__ float2 mnegi(float2 z) { return make_float2(z.y, -z.x); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
__device__ __forceinline__ void dft20p(float2 (&x)[20])
{
    constexpr float C20[13] = {1.0f, 9.510565163e-01f, 8.090169944e-01f, 5.877852523e-01f, 3.090169944e-01f, 0.0f,
                               -3.090169944e-01f, -5.877852523e-01f, -8.090169944e-01f, -9.510565163e-01f, -1.0f,
                               -9.510565163e-01f, -8.090169944e-01f};
    constexpr float S20[13] = {0.0f, 3.090169944e-01f, 5.877852523e-01f, 8.090169944e-01f, 9.510565163e-01f, 1.0f,
                               9.510565163e-01f, 8.090169944e-01f, 5.877852523e-01f, 3.090169944e-01f, 0.0f,
                               -3.090169944e-01f, -5.877852523e-01f};
    float2 A[5][4];
#pragma unroll
    for (int nb = 0; nb < 5; nb++) {
        const float2 s02 = __fadd2_rn(x[nb], x[nb + 10]), d02 = csub(x[nb], x[nb + 10]);
        const float2 s13 = __fadd2_rn(x[nb + 5], x[nb + 15]), t = mnegi(csub(x[nb + 5], x[nb + 15]));
        A[nb][0] = __fadd2_rn(s02, s13);
        A[nb][1] = __fadd2_rn(d02, t);
        A[nb][2] = csub(s02, s13);
        A[nb][3] = csub(d02, t);
    }
#pragma unroll
    for (int nb = 1; nb < 5; nb++)
#pragma unroll
        for (int ka = 1; ka < 4; ka++) A[nb][ka] = cmul(A[nb][ka], make_float2(C20[nb * ka], -S20[nb * ka]));
    const float2 c1 = make_float2(0.30901699437494742f, 0.30901699437494742f);
    const float2 c2 = make_float2(-0.80901699437494742f, -0.80901699437494742f);
    const float2 s1 = make_float2(0.95105651629515357f, 0.95105651629515357f);
    const float2 s2 = make_float2(0.58778525229247313f, 0.58778525229247313f);
    const float2 ms1 = make_float2(-0.95105651629515357f, -0.95105651629515357f);
#pragma unroll
    for (int ka = 0; ka < 4; ka++) {
        const float2 a0 = A[0][ka], a1 = A[1][ka], a2 = A[2][ka], a3 = A[3][ka], a4 = A[4][ka];
        const float2 t1 = __fadd2_rn(a1, a4), t2 = __fadd2_rn(a2, a3), u1 = csub(a1, a4), u2 = csub(a2, a3);
        const float2 r1 = __ffma2_rn(t2, c2, __ffma2_rn(t1, c1, a0));
        const float2 r2 = __ffma2_rn(t2, c1, __ffma2_rn(t1, c2, a0));
        // -i (s1 u1 + s2 u2) and -i (s2 u1 - s1 u2)
        const float2 w1 = mnegi(__ffma2_rn(u2, s2, __fmul2_rn(u1, s1)));
        const float2 w2 = mnegi(__ffma2_rn(u2, ms1, __fmul2_rn(u1, s2)));
        x[ka] = __fadd2_rn(a0, __fadd2_rn(t1, t2));
        x[4 + ka] = __fadd2_rn(r1, w1);
        x[16 + ka] = csub(r1, w1);
        x[8 + ka] = __fadd2_rn(r2, w2);
        x[12 + ka] = csub(r2, w2);
    }
}

__device__ __forceinline__ long long reflect_index(long long j, long long n)
{
    if (n <= 1) return 0;
    const long long p = 2 * (n - 1);
    j %= p;
    if (j < 0) j += p;
    if (j >= n) j = p - j;
    return j;
}

// The log-mel kernel (every log-mel launch of the library).
// Four CTAs of 160 threads per SM walk the (clip, 16-frame block) items of
// the launch, 5 barriers per item.  Thread t takes pair tp = t % 8 and row or
// column tj = t / 8 in every transform phase, so a warp covers 8 pairs x 4
// columns and its shared-memory accesses spread over the banks.
//  pass 1: 20-point DFT over n2 of the windowed samples tj + 20 n2 of both
//          frames of pair tp (frame a real, frame b imaginary), times the
//          400-point twiddle w^(tj k2), into row tj of the pair's buffer
//          (row pitch 20: Z[20 k1 + k2] ends up at element 20 k1 + k2);
//          the block's PCM span is then dead, and the next block's span is
//          fetched into it with cp.async while this block finishes (blocks
//          at the clip ends copy each sample from its reflected source, so
//          no block waits on a synchronous load);
//  pass 2: 20-point DFT over the rows of column tj, in place;
//  power:  bins k = tj + 20 i of both frames from Z[k] and Z[400 - k]; the
//          power pair (a, b) replaces Z[k] in place (the locations a thread
//          reads are its own, so the phase needs no inner barrier);
//  mel:    lane = frame (16), the two half-warps take the even and odd bins
//          of the same group of 4 filters (one shuffle adds them), warp w a
//          run of groups balanced by their work; log-mel rows are staged in the
//          pair's dead upper half (Z[k], k > 200), the pair's two rows
//          together, and leave as one bulk copy per pair.
static constexpr int MEL_MAX_CLIPS = 128;  // clips per launch (the host splits larger batches)
static constexpr int MEL4_FRAMES = 16;
static constexpr int MEL4_THREADS = 160;
static constexpr int MEL4_WARPS = MEL4_THREADS / 32;
static constexpr int MEL4_PAIRS = MEL4_FRAMES / 2;
static constexpr int MEL4_SPAN_SAMPLES = 160 * (MEL4_FRAMES - 1) + 400;  // 2800

// A block's PCM span sits in shared memory with 20 unused words after every
// 320 samples (one frame pair): sample s of the span is word mel_span_pad(s).
// Pass-1 thread (tp, tj) reads sample 20 n2 + tj of pair tp, i.e. word
// 340 tp + tj + 20 n2 (+ 20), whose bank is 20 tp + tj + 20 n2 (mod 32):
// distinct across a warp's 8 pairs x 4 columns.
__host__ __device__ constexpr int mel_span_pad(int s) { return s + 20 * (s / 320); }
static constexpr int MEL4_SPAN = mel_span_pad(MEL4_SPAN_SAMPLES - 1) + 1;  // 2960 words
// Pair pitch of the exchange buffer (float2): 402 = 4 words mod 32 between
// consecutive pairs, so a half-warp's 8 pairs x 2 columns hit distinct banks.
static constexpr int MEL4_YP = 402;
static constexpr int MEL4_STAGE = 416;  // float offset of the staged log-mel rows inside a pair (Z[208] on; 16-byte aligned)

// The filterbank runs over groups of 4 consecutive filters (32 groups); a
// warp takes a contiguous run of groups, balanced by their work.  Group g:
// lo[j] = first bin of filter 4 g + j, nit = bin pairs to visit (the widest
// filter's bins, two per step: one per half-warp), and w4[woff + 2 it + h] =
// the four filters' weights of bin lo[j] + 2 it + h (zero past a filter's
// last bin).
static constexpr int MEL4_GROUPS = 32;
static constexpr int MEL4_MAXIT = (MEL_BAND + 1) / 2;
struct Mel4Group {
    int lo[4];
    int nit, woff, pad0, pad1;
};

// Constant tables of the kernel, built on the host in their shared-memory
// layout and copied in whole at the start.
struct alignas(16) Mel4Tab {
    float2 tw[20][21];  // w^(n1 k2) at [k2][n1], w = exp(-2 pi i / 400)
    float hann[400];
    Mel4Group grp[MEL4_GROUPS];
    float4 w4[MEL4_GROUPS * MEL4_MAXIT * 2];
    int gpart[8];  // groups of warp w: [gpart[w], gpart[w+1])
};
static_assert(sizeof(Mel4Tab) % 16 == 0, "the tables are copied in 16-byte pieces");

struct Mel4Smem {
    Mel4Tab t;
    alignas(16) float2 y[MEL4_PAIRS][MEL4_YP];  // exchange buffer; 16-byte aligned rows (staged rows are read as float4)
    alignas(16) float xs[MEL4_SPAN];            // the block's PCM span (padded); cp.async target
    int first_block[MEL_MAX_CLIPS + 1];
    int scan[MEL4_WARPS];
    float wmax[MEL4_WARPS];
};

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// shared to global memory by the async proxy, in this thread's bulk group.
__device__ __forceinline__ void bulk_store(void *gmem_dst, const void *smem_src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst), "r"(smem_u32(smem_src)),
                 "r"(bytes)
                 : "memory");
}

// Locate item `item` among the clips' blocks: returns false past the end.
__device__ __forceinline__ bool mel4_item(const int *first_block, const MelClip *clips, int n_clips, int item, int &c,
                                          int &frame0, int &nf)
{
    if (item >= first_block[n_clips]) return false;
    int lo = 0, hi = n_clips - 1;  // the last clip whose first block is <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (first_block[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    c = lo;
    const MelClip &cl = clips[c];
    frame0 = cl.f_begin + MEL4_FRAMES * (item - first_block[c]);
    nf = min(MEL4_FRAMES, cl.f_end - frame0);
    return true;
}

// Whether the span of a block lies inside the clip and can be copied as is.
__device__ __forceinline__ bool mel_span_interior(const MelClip &cl, int frame0, int nf)
{
    const long long s0 = 160LL * frame0 - 200;
    return s0 >= 0 && s0 + 160LL * (nf - 1) + 400 <= cl.n && ((reinterpret_cast<uintptr_t>(cl.pcm) & 15) == 0);
}

__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gmem_src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}

// Starts the asynchronous copy of the PCM span of frames frame0 .. frame0 +
// nf - 1 into xs (padded layout): 16-byte pieces when the span lies inside
// the clip, else one 4-byte copy per sample from its reflect-padded source.
template <int THREADS>
__device__ __forceinline__ void mel_span_fetch(float *xs, const MelClip &cl, int frame0, int nf, int tid)
{
    const long long s0 = 160LL * frame0 - 200;
    const int span = 160 * (nf - 1) + 400;
    if (mel_span_interior(cl, frame0, nf)) {
        const float4 *src = reinterpret_cast<const float4 *>(cl.pcm + s0);
        for (int i = tid; i < span / 4; i += THREADS) cp_async16(reinterpret_cast<float4 *>(xs) + i + 5 * (i / 80), src + i);
    } else {
        for (int i = tid; i < span; i += THREADS) {
            long long j = s0 + i;
            if (j < 0 || j >= cl.n) j = reflect_index(j, cl.n);
            cp_async4(xs + mel_span_pad(i), cl.pcm + j);
        }
    }
}

__global__ void __launch_bounds__(MEL4_THREADS, 4) logmel4_kernel(const MelClip *__restrict__ clips, int n_clips,
                                                                  const Mel4Tab *__restrict__ tab,
                                                                  float *__restrict__ out, int *gmax_ord,
                                                                  int write_out)
{
    extern __shared__ __align__(16) uint8_t mel4_smem[];
    Mel4Smem &S = *reinterpret_cast<Mel4Smem *>(mel4_smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the tables: one round of 16-byte copies
    for (int i = tid; i < (int)(sizeof(Mel4Tab) / 16); i += MEL4_THREADS)
        cp_async16(reinterpret_cast<float4 *>(&S.t) + i, reinterpret_cast<const float4 *>(tab) + i);
    cp_async_commit();
    grid_dep_wait();
    grid_dep_launch();
    // blocks per clip -> prefix (thread c takes clip c; n_clips <= MEL_MAX_CLIPS <= MEL4_THREADS)
    {
        int nb = 0;
        if (tid < n_clips) {
            const int f = clips[tid].f_end - clips[tid].f_begin;
            nb = f > 0 ? (f + MEL4_FRAMES - 1) / MEL4_FRAMES : 0;
        }
        int incl = nb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) S.scan[warp] = incl;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; w++) base += S.scan[w];
        if (tid <= n_clips) S.first_block[tid] = base + incl - nb;  // exclusive prefix; [n_clips] = total
        cp_async_wait_all();
        __syncthreads();
    }

    // span loader: locates `item` (nc < 0 past the end) and starts the
    // asynchronous copy of its span
    auto prefetch = [&](int item, int &nc, int &nframe0, int &nnf) {
        if (!mel4_item(S.first_block, clips, n_clips, item, nc, nframe0, nnf)) {
            nc = -1;
            return;
        }
        mel_span_fetch<MEL4_THREADS>(S.xs, clips[nc], nframe0, nnf, tid);
    };

    const float log10_2 = 0.30102999566398120f;
    const bool out_aligned = (reinterpret_cast<uintptr_t>(out) & 15) == 0;
    const int tp = tid & 7, tj = tid >> 3;
    const float *hw = S.t.hann + tj;  // window value of sample tj + 20 n2: hw[20 n2]
    int c, frame0, nf;
    prefetch(blockIdx.x, c, frame0, nf);
    cp_async_commit();
    for (int item = blockIdx.x; c >= 0; item += gridDim.x) {
        const MelClip cl = clips[c];
        cp_async_wait_all();
        if (write_out && out_aligned && tid < MEL4_PAIRS) bulk_wait_read();  // the previous rows have left the staging area
        __syncthreads();  // B0: span in place; staging area free

        const int npairs = (nf + 1) / 2;
        float2 *Y = S.y[tp];
        if (tp < npairs) {
            // pass 1 (frame 2 tp starts at span sample 320 tp, frame 2 tp + 1 at 320 tp + 160)
            const bool has_b = 2 * tp + 1 < nf;
            const float *xa = S.xs + 340 * tp + tj, *xb = xa + 160;
            float2 v[20];
#pragma unroll
            for (int n2 = 0; n2 < 20; n2++) {
                const float a = xa[20 * n2 + (n2 >= 16 ? 20 : 0)];
                const float b = has_b ? xb[20 * n2 + (n2 >= 8 ? 20 : 0)] : 0.0f;
                v[n2] = make_float2(hw[20 * n2] * a, hw[20 * n2] * b);
            }
            dft20p(v);
            float2 *yr = Y + tj * 20;
            yr[0] = v[0];
#pragma unroll
            for (int k2 = 1; k2 < 20; k2++) yr[k2] = cmul(v[k2], S.t.tw[k2][tj]);  // w^0 = 1 exactly for tj = 0
        }
        __syncthreads();  // B1: pass-1 rows written; the span is dead
        int c_next, frame0_next, nf_next;
        prefetch(item + gridDim.x, c_next, frame0_next, nf_next);
        cp_async_commit();
        if (tp < npairs) {
            // pass 2: 20-point DFT over n1 -> Z[20 k1 + tj], in place (own column)
            float2 v[20];
#pragma unroll
            for (int n1 = 0; n1 < 20; n1++) v[n1] = Y[n1 * 20 + tj];
            dft20p(v);
#pragma unroll
            for (int k1 = 0; k1 < 20; k1++) Y[k1 * 20 + tj] = v[k1];
        }
        __syncthreads();  // B2: the pair's spectrum Z is complete
        if (tp < npairs) {
            // X_a[k] = (Z[k] + conj Z[400-k]) / 2, X_b[k] = (Z[k] - conj Z[400-k]) / 2i, k = tj + 20 i
            float2 zk[11], zn[11];
#pragma unroll
            for (int i = 0; i < 11; i++) {
                const int k = tj + 20 * i;
                if (k <= 200) {
                    zk[i] = Y[k];
                    zn[i] = Y[k == 0 ? 0 : 400 - k];
                }
            }
#pragma unroll
            for (int i = 0; i < 11; i++) {
                const int k = tj + 20 * i;
                if (k <= 200) {
                    const float ar = zk[i].x + zn[i].x, ai = zk[i].y - zn[i].y;
                    const float br = zk[i].y + zn[i].y, bi = zk[i].x - zn[i].x;
                    Y[k] = make_float2(0.25f * (ar * ar + ai * ai), 0.25f * (br * br + bi * bi));
                }
            }
        }
        __syncthreads();  // B3: power of every frame in place: frame f, bin k at float 2 k + (f & 1) of pair f / 2
        float lmax = -INFINITY;
        {
            // lane = frame f, half-warp h takes bins lo + 2 it + h of each filter
            // of the group; bins a little past a filter's last one carry zero
            // weight and read finite spectrum values (Z[k], k > 200, is written
            // by pass 2 of every active pair)
            const int f = lane & 15, h = lane >> 4;
            const float *P = reinterpret_cast<const float *>(S.y[f >> 1]) + (f & 1) + 2 * h;
            float *ost = reinterpret_cast<float *>(S.y[f >> 1]) + MEL4_STAGE + 128 * (f & 1);
            const int g1 = S.t.gpart[warp + 1];
            for (int g = S.t.gpart[warp]; g < g1; g++) {
                const Mel4Group G = S.t.grp[g];
                const float *p0 = P + 2 * G.lo[0], *p1 = P + 2 * G.lo[1], *p2 = P + 2 * G.lo[2], *p3 = P + 2 * G.lo[3];
                const float4 *wv = S.t.w4 + G.woff + h;
                float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
                for (int it = 0; it < MEL4_MAXIT; it++) {
                    if (it >= G.nit) break;
                    const float4 w = wv[2 * it];
                    a0 = fmaf(w.x, p0[4 * it], a0);
                    a1 = fmaf(w.y, p1[4 * it], a1);
                    a2 = fmaf(w.z, p2[4 * it], a2);
                    a3 = fmaf(w.w, p3[4 * it], a3);
                }
                a0 += __shfl_xor_sync(0xffffffffu, a0, 16);
                a1 += __shfl_xor_sync(0xffffffffu, a1, 16);
                a2 += __shfl_xor_sync(0xffffffffu, a2, 16);
                a3 += __shfl_xor_sync(0xffffffffu, a3, 16);
                // half 0 emits filters 4 g, 4 g + 1, half 1 filters 4 g + 2, 4 g + 3
                const float e0 = h ? a2 : a0, e1 = h ? a3 : a1;
                const float r0 = __log2f(fmaxf(e0, 1e-10f)) * log10_2, r1 = __log2f(fmaxf(e1, 1e-10f)) * log10_2;
                if (f < nf) lmax = fmaxf(lmax, fmaxf(r0, r1));
                const int m = 4 * g + 2 * h;
                ost[m] = r0;
                ost[m + 1] = r1;
            }
        }
        if (cl.gslot >= 0) {
            for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
            if (lane == 0) S.wmax[warp] = lmax;
        }
        fence_async_smem();  // the staged rows are read by the bulk copies below
        __syncthreads();  // B4: staged rows and warp maxima written
        if (write_out && out_aligned) {
            if (tid < npairs) {
                // frames 2 tid, 2 tid + 1: consecutive output rows, staged back to back
                const long long row = cl.out_row0 + (frame0 - cl.f_begin) + 2 * tid;
                const uint32_t bytes = (2 * tid + 1 < nf ? 2 : 1) * 128 * 4;
                bulk_store(out + (size_t)row * 128, reinterpret_cast<const float *>(S.y[tid]) + MEL4_STAGE, bytes);
                bulk_commit();
            }
        } else if (write_out) {  // an output buffer without 16-byte alignment: plain stores
            const long long out_row = cl.out_row0 + (frame0 - cl.f_begin);
            for (int i = tid; i < nf * 128; i += MEL4_THREADS) {
                const int f = i >> 7;
                out[(size_t)(out_row + f) * 128 + (i & 127)] =
                    reinterpret_cast<const float *>(S.y[f >> 1])[MEL4_STAGE + 128 * (f & 1) + (i & 127)];
            }
        }
        if (cl.gslot >= 0 && tid == 0) {
            float m = S.wmax[0];
            for (int i = 1; i < MEL4_WARPS; i++) m = fmaxf(m, S.wmax[i]);
            atomicMax(gmax_ord + cl.gslot, float_to_ordered(m));
        }
        c = c_next;
        frame0 = frame0_next;
        nf = nf_next;
    }
    cp_async_wait_all();
    if (write_out && out_aligned && tid < MEL4_PAIRS) bulk_wait_all();
}

// In-place Whisper normalisation of rows [n_rows][128]: (max(x, g - 8) + 4) / 4.
__global__ void mel_normalize_kernel(float *mel, long long count, const int *gmax_ord)
{
    const float g = ordered_to_float(*gmax_ord) - 8.0f;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count;
         i += (long long)gridDim.x * blockDim.x)
        mel[i] = (fmaxf(mel[i], g) + 4.0f) * 0.25f;
}

// gmax slots from caller-given device floats (or -inf to start an atomicMax).
__global__ void gmax_init_kernel(int *gmax_ord, const float *const *src, int n)
{
    grid_dep_wait();
    grid_dep_launch();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) gmax_ord[i] = float_to_ordered(src[i] ? *src[i] : -INFINITY);
}

__global__ void gmax_export_kernel(const int *gmax_ord, float *dst)
{
    if (threadIdx.x == 0 && blockIdx.x == 0) *dst = ordered_to_float(*gmax_ord);
}

}  // namespace moss
