// Whisper-style log-mel front end (fp32, CUDA cores).
//
// One CTA takes a block of up to 32 consecutive frames of one clip.  The PCM
// span those frames cover (160*31 + 400 samples) is read once, coalesced, into
// shared memory, with reflect padding applied only at the true clip ends.  Each
// warp then transforms two frames at a time: frame a as the real part and
// frame b as the imaginary part of one 400-point complex DFT, computed as
// 20 x 20 (two passes of 20-point DFTs, each a 4-point and a 5-point stage,
// with the 400-point twiddles between the passes).  The two real spectra are
// separated with X_a[k] = (Z[k] + conj Z[-k]) / 2, X_b[k] = (Z[k] - conj Z[-k]) / 2i,
// squared, pushed through the banded mel filterbank, and log10'd.  The block's
// maximum goes to the clip's maximum with one ordered-integer atomicMax.
#pragma once

#include "common.cuh"

namespace moss {

static constexpr int MEL_FRAMES_PER_BLOCK = 32;
static constexpr int MEL_BAND = 16;  // max nonzero FFT bins of one mel filter
static constexpr int MEL_SPAN = 160 * (MEL_FRAMES_PER_BLOCK - 1) + 400;

// One clip's frame range for a logmel launch.  Block (x, y) of the grid
// takes frames f_begin + 32x .. of clip y; frame f goes to output row
// out_row0 + (f - f_begin).  gslot >= 0 names the per-clip maximum this
// range folds into (atomicMax); -1 folds into nothing.
struct MelClip {
    const float *pcm;
    long long n;
    long long out_row0;
    int f_begin, f_end;
    int gslot;
    int pad;
};

// Device tables shared by every mel launch (filled at create).
struct MelTables {
    float2 tw400[400];            // exp(-2 pi i k / 400)
    float hann[400];              // periodic Hann
    int band_lo[128];             // first nonzero bin of each filter
    float band_w[128][MEL_BAND];  // filter weights on bins band_lo .. band_lo+15
};

// Shared memory of one logmel CTA (dynamic; about 74 KB).
struct MelSmem {
    float2 tw[400];
    float2 zbuf[8][400];   // per warp: the 20 x 20 exchange, then Z
    float xs[MEL_SPAN];    // the PCM span of the block
    float hann[400];
    int band_lo[128];
    float band_w[128][MEL_BAND];
    float pw[8][2][204];   // per warp: power of frames a and b
    float wmax[8];
};

__device__ __forceinline__ float2 cmul(float2 a, float2 b)
{
    return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

// 20-point DFT in registers: X[k] = sum_n x[n] exp(-2 pi i n k / 20).
// n = nb + 5 na, k = 4 kb + ka:  4-point DFTs over na, twiddle
// exp(-2 pi i nb ka / 20), then 5-point DFTs over nb.
__device__ __forceinline__ void dft20(float2 (&x)[20], const float2 *tw400)
{
    float2 A[5][4];
#pragma unroll
    for (int nb = 0; nb < 5; nb++) {
        float2 x0 = x[nb], x1 = x[nb + 5], x2 = x[nb + 10], x3 = x[nb + 15];
        float2 s02 = make_float2(x0.x + x2.x, x0.y + x2.y), d02 = make_float2(x0.x - x2.x, x0.y - x2.y);
        float2 s13 = make_float2(x1.x + x3.x, x1.y + x3.y), d13 = make_float2(x1.x - x3.x, x1.y - x3.y);
        // W4 = -i: (-i) * d13 = (d13.y, -d13.x)
        A[nb][0] = make_float2(s02.x + s13.x, s02.y + s13.y);
        A[nb][1] = make_float2(d02.x + d13.y, d02.y - d13.x);
        A[nb][2] = make_float2(s02.x - s13.x, s02.y - s13.y);
        A[nb][3] = make_float2(d02.x - d13.y, d02.y + d13.x);
    }
#pragma unroll
    for (int nb = 1; nb < 5; nb++)
#pragma unroll
        for (int ka = 1; ka < 4; ka++) A[nb][ka] = cmul(A[nb][ka], tw400[20 * nb * ka]);
    // 5-point DFT with c1 = cos(2pi/5), c2 = cos(4pi/5), s1 = sin(2pi/5), s2 = sin(4pi/5)
    const float c1 = 0.30901699437494742f, c2 = -0.80901699437494742f;
    const float s1 = 0.95105651629515357f, s2 = 0.58778525229247313f;
#pragma unroll
    for (int ka = 0; ka < 4; ka++) {
        float2 a0 = A[0][ka], a1 = A[1][ka], a2 = A[2][ka], a3 = A[3][ka], a4 = A[4][ka];
        float2 t1 = make_float2(a1.x + a4.x, a1.y + a4.y), t2 = make_float2(a2.x + a3.x, a2.y + a3.y);
        float2 u1 = make_float2(a1.x - a4.x, a1.y - a4.y), u2 = make_float2(a2.x - a3.x, a2.y - a3.y);
        float2 r1 = make_float2(a0.x + c1 * t1.x + c2 * t2.x, a0.y + c1 * t1.y + c2 * t2.y);
        float2 r2 = make_float2(a0.x + c2 * t1.x + c1 * t2.x, a0.y + c2 * t1.y + c1 * t2.y);
        // -i * (s1 u1 + s2 u2) and -i * (s2 u1 - s1 u2)
        float2 i1 = make_float2(s1 * u1.x + s2 * u2.x, s1 * u1.y + s2 * u2.y);
        float2 i2 = make_float2(s2 * u1.x - s1 * u2.x, s2 * u1.y - s1 * u2.y);
        x[ka] = make_float2(a0.x + t1.x + t2.x, a0.y + t1.y + t2.y);
        x[4 + ka] = make_float2(r1.x + i1.y, r1.y - i1.x);
        x[16 + ka] = make_float2(r1.x - i1.y, r1.y + i1.x);
        x[8 + ka] = make_float2(r2.x + i2.y, r2.y - i2.x);
        x[12 + ka] = make_float2(r2.x - i2.y, r2.y + i2.x);
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

// out: rows of 128 fp32 log10 mel values (not normalised) when write_out.
// gmax_ord: per-clip ordered-int maxima (atomicMax) when do_max.
__global__ void __launch_bounds__(256) logmel_kernel(const MelClip *__restrict__ clips,
                                                     const MelTables *__restrict__ tab,
                                                     float *__restrict__ out, int *gmax_ord,
                                                     int write_out)
{
    extern __shared__ __align__(16) uint8_t mel_smem[];
    MelSmem &S = *reinterpret_cast<MelSmem *>(mel_smem);
    float *xs = S.xs;
    float2 *tw = S.tw;
    float *hann = S.hann;
    int *band_lo = S.band_lo;
    float (*band_w)[MEL_BAND] = S.band_w;
    float2 (*zbuf)[400] = S.zbuf;
    float (*pw)[2][204] = S.pw;
    float *wmax = S.wmax;

    const MelClip clip = clips[blockIdx.y];
    struct { int frame0, nframes; long long out_row; } blk;
    blk.frame0 = clip.f_begin + MEL_FRAMES_PER_BLOCK * blockIdx.x;
    if (blk.frame0 >= clip.f_end) return;
    blk.nframes = min(MEL_FRAMES_PER_BLOCK, clip.f_end - blk.frame0);
    blk.out_row = clip.out_row0 + (blk.frame0 - clip.f_begin);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int i = tid; i < 400; i += 256) {
        tw[i] = tab->tw400[i];
        hann[i] = tab->hann[i];
    }
    for (int i = tid; i < 128; i += 256) band_lo[i] = tab->band_lo[i];
    for (int i = tid; i < 128 * MEL_BAND; i += 256) band_w[i / MEL_BAND][i % MEL_BAND] = tab->band_w[i / MEL_BAND][i % MEL_BAND];

    const long long s0 = 160LL * blk.frame0 - 200;
    const int span = 160 * (blk.nframes - 1) + 400;
    const bool interior = s0 >= 0 && s0 + span <= clip.n;
    if (interior && (s0 & 3) == 0 && ((reinterpret_cast<uintptr_t>(clip.pcm) & 15) == 0)) {
        const float4 *src = reinterpret_cast<const float4 *>(clip.pcm + s0);
        for (int i = tid; i < (span + 3) / 4; i += 256) {
            if (4 * i + 3 < span) {
                float4 v = __ldg(src + i);
                xs[4 * i] = v.x;
                xs[4 * i + 1] = v.y;
                xs[4 * i + 2] = v.z;
                xs[4 * i + 3] = v.w;
            } else {
                for (int j = 4 * i; j < span; j++) xs[j] = clip.pcm[s0 + j];
            }
        }
    } else {
        for (int i = tid; i < span; i += 256) xs[i] = __ldg(clip.pcm + reflect_index(s0 + i, clip.n));
    }
    __syncthreads();

    float lmax = -INFINITY;
    const int npairs = (blk.nframes + 1) / 2;
    for (int pr = warp; pr < npairs; pr += 8) {
        const int fa = 2 * pr, fb = 2 * pr + 1;
        const bool has_b = fb < blk.nframes;
        const float *xa = xs + 160 * fa;
        const float *xb = xs + 160 * (has_b ? fb : fa);
        float2 *z = zbuf[warp];
        // pass 1: lane n1 < 20 takes samples n1 + 20 n2
        if (lane < 20) {
            float2 v[20];
#pragma unroll
            for (int n2 = 0; n2 < 20; n2++) {
                const int nidx = lane + 20 * n2;
                const float w = hann[nidx];
                v[n2] = make_float2(w * xa[nidx], has_b ? w * xb[nidx] : 0.0f);
            }
            dft20(v, tw);
#pragma unroll
            for (int k2 = 0; k2 < 20; k2++) {
                float2 t = k2 == 0 || lane == 0 ? v[k2] : cmul(v[k2], tw[(lane * k2) % 400]);
                z[lane * 20 + k2] = t;
            }
        }
        __syncwarp();
        // pass 2: lane k2 < 20 takes column k2 -> Z[20 k1 + k2]
        float2 v2[20];
        if (lane < 20) {
#pragma unroll
            for (int n1 = 0; n1 < 20; n1++) v2[n1] = z[n1 * 20 + lane];
            dft20(v2, tw);
        }
        __syncwarp();
        if (lane < 20) {
#pragma unroll
            for (int k1 = 0; k1 < 20; k1++) z[20 * k1 + lane] = v2[k1];
        }
        __syncwarp();
        // split the two real spectra and take the power
        for (int k = lane; k <= 200; k += 32) {
            const float2 zk = z[k], zn = z[(400 - k) % 400];
            const float ar = 0.5f * (zk.x + zn.x), ai = 0.5f * (zk.y - zn.y);
            const float br = 0.5f * (zk.y + zn.y), bi = -0.5f * (zk.x - zn.x);
            pw[warp][0][k] = ar * ar + ai * ai;
            pw[warp][1][k] = br * br + bi * bi;
        }
        __syncwarp();
        // mel: lane handles filters 4 lane .. 4 lane + 3 of both frames
#pragma unroll
        for (int f = 0; f < 2; f++) {
            if (f == 1 && !has_b) break;
            float r[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int m = 4 * lane + j;
                const int lo = band_lo[m];
                float acc = 0.0f;
#pragma unroll
                for (int b = 0; b < MEL_BAND; b++) {
                    const int k = lo + b;
                    acc += band_w[m][b] * (k <= 200 ? pw[warp][f][k] : 0.0f);
                }
                r[j] = log10f(fmaxf(acc, 1e-10f));
                lmax = fmaxf(lmax, r[j]);
            }
            if (write_out) {
                const int frame = f == 0 ? fa : fb;
                float4 *dst = reinterpret_cast<float4 *>(out + (size_t)(blk.out_row + frame) * 128) + lane;
                *dst = make_float4(r[0], r[1], r[2], r[3]);
            }
        }
        __syncwarp();
    }
    if (clip.gslot >= 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
        if (lane == 0) wmax[warp] = lmax;
        __syncthreads();
        if (tid == 0) {
            float m = wmax[0];
            for (int i = 1; i < 8; i++) m = fmaxf(m, wmax[i]);
            atomicMax(gmax_ord + clip.gslot, float_to_ordered(m));
        }
    }
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
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) gmax_ord[i] = float_to_ordered(src[i] ? *src[i] : -INFINITY);
}

__global__ void gmax_export_kernel(const int *gmax_ord, float *dst)
{
    if (threadIdx.x == 0 && blockIdx.x == 0) *dst = ordered_to_float(*gmax_ord);
}

}  // namespace moss
