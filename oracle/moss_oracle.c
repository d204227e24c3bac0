/*
 * Oracle: a plain, slow CPU restatement of the audio-encoder forward of the
 * MOSS-Audio / MOSS-Transcribe family (Qwen3-Omni AuT tower).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is used by the tests, by the smoke
 * check and by the benchmark's CPU-baseline leg.  The CUDA library never
 * includes, links or calls it, and it shares no code with the CUDA library.
 *
 * Precision: activations are stored in fp32 (the pages validate against an
 * "fp32 CPU reference"), every sum and every transcendental function is
 * evaluated in fp64, and weights are the bf16 values of the blob widened to
 * fp32.  The front end (STFT, power, mel, log) is fp64 throughout and its
 * result is stored as fp32.
 *
 * Sources (page title, section):
 *  - "MOSS-Transcribe-preview-2B - GGUF", "Architecture" table: the layer
 *    widths, the 3 x Conv2D stride-2 stem 1->480->480->480, conv_out
 *    480*16=7680->1280 without bias, sinusoidal positions, 32 pre-LN layers
 *    d=1280, 20 heads x 64, FFN 5120, windowed (block-diagonal) attention,
 *    ln_post -> proj1 -> GELU -> proj2 (1280->2048), SwiGLU adapter
 *    2048->8192->2048; the "Audio" row: 16 kHz mono, 128 mel bins, n_fft 400,
 *    hop 160, matching the Whisper feature extractor.
 *  - same page, "Non-obvious gotchas" item 2: the trailing STFT frame is
 *    dropped, so a clip of n samples has exactly n/160 frames.
 *  - "MOSS-Music-8B-Instruct-GGUF", "Conversion provenance": inv_timescales is
 *    recomputed, so positions are computed, not stored; the encoder is
 *    prompt-independent ("Usage in HOT-Step").
 *  - "Ossicle-4B", "Long Audio": 64 s pieces give log-mel identical to the
 *    whole clip, so the log-mel floor uses the whole-clip maximum.
 *  - The workload statement fixes the front-end details the pages leave to
 *    "Whisper": periodic Hann, Slaney mel 0-8 kHz, log10 clamp 1e-10, floor at
 *    max-8, (x+4)/4; 3x3 kernels with GELU; 800-frame chunks zero-padded at
 *    the tail; 100-token attention windows; N(0,1/fan_in) weights.
 *
 * Readings where the pages are silent (each one also listed in the design
 * notes): centred frames with reflect padding at the true clip ends
 * (periodic reflection when the clip is shorter than the pad); |X|^2 power;
 * exact-erf GELU; LayerNorm eps 1e-5 with biased variance; conv padding 1;
 * conv_out input index c*16+f; positions restart at 0 in every 800-frame
 * chunk, 640 sin then 640 cos channels, inv_timescale_i =
 * exp(-i*ln(10000)/639); attention scale 1/sqrt(64); SiLU on the gate branch.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define SR 16000
#define N_FFT 400
#define HOP 160
#define PAD (N_FFT / 2)
#define N_BINS (N_FFT / 2 + 1)
#define N_MELS 128
#define CHUNK_FRAMES 800
#define D 1280
#define N_HEADS 20
#define HEAD_DIM 64
#define D_FFN 5120
#define C_STEM 480
#define F_STEM 16
#define D_OUT 2048
#define D_ADP 8192
#define LN_EPS 1e-5

static double bf(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float bff(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ counts */

/* Frames of a clip: centred STFT gives n/hop + 1 frames, the trailing one is
 * dropped ("gotcha" 2), so n // 160. */
int64_t oracle_num_frames(int64_t n_samples)
{
    return n_samples <= 0 ? 0 : n_samples / HOP;
}

/* Tokens of one chunk of F frames: three convs of kernel 3, stride 2,
 * padding 1 each map a length L to floor((L + 2 - 3) / 2) + 1. */
int64_t oracle_chunk_tokens(int64_t frames)
{
    int64_t L = frames;
    for (int i = 0; i < 3; i++) L = L <= 0 ? 0 : (L + 2 - 3) / 2 + 1;
    return L;
}

int64_t oracle_num_chunks(int64_t n_samples)
{
    int64_t F = oracle_num_frames(n_samples);
    return (F + CHUNK_FRAMES - 1) / CHUNK_FRAMES;
}

/* Tokens of a clip: the sum over 800-frame chunks of the chunk's tokens. */
int64_t oracle_num_tokens(int64_t n_samples)
{
    int64_t F = oracle_num_frames(n_samples), T = 0;
    for (int64_t s = 0; s < F; s += CHUNK_FRAMES) {
        int64_t fc = F - s < CHUNK_FRAMES ? F - s : CHUNK_FRAMES;
        T += oracle_chunk_tokens(fc);
    }
    return T;
}

/* ---------------------------------------------------------------- front end */

/* Periodic Hann of length N_FFT: w[n] = 0.5 - 0.5 cos(2 pi n / N). */
void oracle_hann(double *w)
{
    for (int n = 0; n < N_FFT; n++) w[n] = 0.5 - 0.5 * cos(2.0 * M_PI * n / N_FFT);
}

static double hz_to_mel_slaney(double f)
{
    const double f_sp = 200.0 / 3.0, min_log_hz = 1000.0;
    const double min_log_mel = min_log_hz / f_sp, logstep = log(6.4) / 27.0;
    if (f < min_log_hz) return f / f_sp;
    return min_log_mel + log(f / min_log_hz) / logstep;
}

static double mel_to_hz_slaney(double m)
{
    const double f_sp = 200.0 / 3.0, min_log_hz = 1000.0;
    const double min_log_mel = min_log_hz / f_sp, logstep = log(6.4) / 27.0;
    if (m < min_log_mel) return f_sp * m;
    return min_log_hz * exp(logstep * (m - min_log_mel));
}

/* Slaney-style mel filterbank, 128 triangles over 0..8 kHz, area-normalised:
 * 130 edge frequencies equally spaced on the Slaney mel scale; filter m rises
 * linearly from edge m to edge m+1 and falls to edge m+2, evaluated at the FFT
 * bin frequencies k*SR/N_FFT, and is scaled by 2/(f[m+2]-f[m]). */
void oracle_mel_filters(double *W /* [N_MELS][N_BINS] */)
{
    double edges[N_MELS + 2];
    double m_lo = hz_to_mel_slaney(0.0), m_hi = hz_to_mel_slaney(SR / 2.0);
    for (int i = 0; i < N_MELS + 2; i++)
        edges[i] = mel_to_hz_slaney(m_lo + (m_hi - m_lo) * i / (N_MELS + 1));
    for (int m = 0; m < N_MELS; m++) {
        double norm = 2.0 / (edges[m + 2] - edges[m]);
        for (int k = 0; k < N_BINS; k++) {
            double f = (double)k * SR / N_FFT;
            double up = (f - edges[m]) / (edges[m + 1] - edges[m]);
            double down = (edges[m + 2] - f) / (edges[m + 2] - edges[m + 1]);
            double v = up < down ? up : down;
            W[m * N_BINS + k] = (v > 0.0 ? v : 0.0) * norm;
        }
    }
}

/* Reflect padding about the clip ends (the sample at the end is not
 * repeated); indices further out than one clip length keep reflecting, which
 * is the periodic extension with period 2(n-1). */
static int64_t reflect_index(int64_t j, int64_t n)
{
    if (n == 1) return 0;
    int64_t p = 2 * (n - 1);
    j %= p;
    if (j < 0) j += p;
    if (j >= n) j = p - j;
    return j;
}

/* Power spectrum |X_k|^2, k = 0..200, of frame t (centred on sample 160 t),
 * by the direct O(N^2) DFT of the Hann-windowed frame. */
void oracle_frame_power(const float *pcm, int64_t n, int64_t t, double *P)
{
    double w[N_FFT], c[N_FFT], s[N_FFT], x[N_FFT];
    oracle_hann(w);
    for (int m = 0; m < N_FFT; m++) {
        c[m] = cos(2.0 * M_PI * m / N_FFT);
        s[m] = sin(2.0 * M_PI * m / N_FFT);
    }
    for (int i = 0; i < N_FFT; i++)
        x[i] = w[i] * (double)pcm[reflect_index(t * HOP - PAD + i, n)];
    for (int k = 0; k < N_BINS; k++) {
        double re = 0.0, im = 0.0;
        for (int i = 0; i < N_FFT; i++) {
            int m = (int)(((int64_t)k * i) % N_FFT);
            re += x[i] * c[m];
            im -= x[i] * s[m];
        }
        P[k] = re * re + im * im;
    }
}

/* Unnormalised log-mel of frames [f0, f1): log10(max(W P, 1e-10)).
 * out is [(f1 - f0)][128], frame-major. */
void oracle_logmel_raw(const float *pcm, int64_t n, int64_t f0, int64_t f1, float *out)
{
    double *W = (double *)malloc(sizeof(double) * N_MELS * N_BINS);
    oracle_mel_filters(W);
#pragma omp parallel for schedule(static)
    for (int64_t t = f0; t < f1; t++) {
        double P[N_BINS];
        oracle_frame_power(pcm, n, t, P);
        for (int m = 0; m < N_MELS; m++) {
            double acc = 0.0;
            for (int k = 0; k < N_BINS; k++) acc += W[m * N_BINS + k] * P[k];
            out[(t - f0) * N_MELS + m] = (float)log10(acc > 1e-10 ? acc : 1e-10);
        }
    }
    free(W);
}

float oracle_max(const float *x, int64_t count)
{
    float mx = -INFINITY;
    for (int64_t i = 0; i < count; i++) mx = x[i] > mx ? x[i] : mx;
    return mx;
}

/* Whisper normalisation: floor at (global max - 8), then (x + 4) / 4. */
void oracle_normalize(float *mel, int64_t count, float gmax)
{
    double lo = (double)gmax - 8.0;
    for (int64_t i = 0; i < count; i++) {
        double v = mel[i] > lo ? mel[i] : lo;
        mel[i] = (float)((v + 4.0) / 4.0);
    }
}

/* Whole-clip maximum of the unnormalised log-mel. */
float oracle_clip_log_max(const float *pcm, int64_t n)
{
    int64_t F = oracle_num_frames(n);
    if (F == 0) return -INFINITY;
    float *raw = (float *)malloc(sizeof(float) * F * N_MELS);
    oracle_logmel_raw(pcm, n, 0, F, raw);
    float mx = oracle_max(raw, F * N_MELS);
    free(raw);
    return mx;
}

/* Normalised log-mel of the whole clip: out [F][128]; returns the max. */
float oracle_logmel(const float *pcm, int64_t n, float *out)
{
    int64_t F = oracle_num_frames(n);
    if (F == 0) return -INFINITY;
    oracle_logmel_raw(pcm, n, 0, F, out);
    float mx = oracle_max(out, F * N_MELS);
    oracle_normalize(out, F * N_MELS, mx);
    return mx;
}

/* ------------------------------------------------------------ model weights */

typedef struct {
    const uint16_t *ln1_g, *ln1_b, *ln2_g, *ln2_b;
    const uint16_t *bq, *bk, *bv, *bo, *b1, *b2;
    uint16_t *wq_t, *wk_t, *wv_t, *wo_t, *w1_t, *w2_t; /* [in][out] */
    float *sq, *sk, *sv, *s1; /* FP8 models: per-channel scales of q, k, v, fc1 */
} layer_w;

typedef struct oracle_model {
    int n_layers;
    int fp8;            /* q, k, v and fc1 on e4m3 operands */
    int nvfp4;          /* q, k, v and fc1 on NVFP4 operands (sq.. hold the weight tensors' g) */
    float *conv_w_t[3]; /* [in][3][3][out] */
    const uint16_t *conv_b[3];
    int conv_in[3];
    uint16_t *conv_out_t; /* [7680][1280] */
    layer_w *layers;
    const uint16_t *lnp_g, *lnp_b, *bp1, *bp2, *bg, *bu, *bd;
    uint16_t *wp1_t, *wp2_t, *wg_t, *wu_t, *wd_t;
} oracle_model;

/* Transpose a bf16 [out][in] matrix into [in][out]. */
static uint16_t *transpose_bf16(const uint16_t *w, int out, int in)
{
    uint16_t *t = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)out * in);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < in; i++)
        for (int o = 0; o < out; o++) t[(size_t)i * out + o] = w[(size_t)o * in + i];
    return t;
}

/* ------------------------------------------------ 4-bit weight quantisation
 *
 * Page "Ossicle-4B", "Long Audio", note under the table: the 4-bit variant
 * keeps "4-bit weights for the language model and the audio encoder, round to
 * nearest, groups of 128".  Reading (the page gives no more): symmetric
 * round-to-nearest over groups of 128 consecutive input features of each
 * output row; the group's scale is its largest magnitude over 7, so codes lie
 * in [-7, 7] (the 4-bit range [-8, 7] is the clamp); a weight's value in the
 * quantised model is its code times the scale.  The arithmetic is fixed so
 * that two implementations agree bit for bit:
 *   s   = fp32(max |w|) / 7            (fp32 division)
 *   q   = clamp(rint(w / s), -8, 7)    (fp32 division, ties to even; 0 if s = 0)
 *   w'  = bf16(fp32(q * s))            (fp32 product, then to bf16, ties to even)
 * The linear layers of the 32 encoder layers, the encoder head and the adapter
 * are quantised; the conv stem (conv1..conv3 and conv_out) keeps bf16. */

/* Round an fp32 value to the nearest bf16, ties to even (finite inputs). */
static uint16_t bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    const uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* Quantise w [rows][cols] (bf16 bits, cols % 128 == 0) group by group.
 * deq receives w' (bf16 bits); codes (optional) q + 8 in [0, 15]; scales
 * (optional) s per [row][group]. */
void oracle_quant_rtn4(const uint16_t *w, int rows, int cols, uint16_t *deq, uint8_t *codes, float *scales)
{
    const int groups = cols / 128;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; r++)
        for (int g = 0; g < groups; g++) {
            const uint16_t *wg = w + (size_t)r * cols + (size_t)g * 128;
            float amax = 0.0f;
            for (int k = 0; k < 128; k++) {
                const float a = fabsf(bff(wg[k]));
                if (a > amax) amax = a;
            }
            const float s = amax / 7.0f;
            if (scales) scales[(size_t)r * groups + g] = s;
            for (int k = 0; k < 128; k++) {
                float q = 0.0f;
                if (s > 0.0f) {
                    q = rintf(bff(wg[k]) / s);
                    if (q < -8.0f) q = -8.0f;
                    if (q > 7.0f) q = 7.0f;
                }
                const size_t i = (size_t)r * cols + (size_t)g * 128 + k;
                if (codes) codes[i] = (uint8_t)((int)q + 8);
                const float v = q * s;
                deq[i] = bf16_rne(v);
            }
        }
}

/* ------------------------------------------------ FP8 (e4m3) GEMM operands
 *
 * Page "Ossicle-4B", "Quantized: NVFP4 and INT4 in vLLM": the low-precision
 * builds quantise weights and activations of the audio encoder and run on
 * Blackwell's low-precision tensor cores.  Reading for an FP8 encoder (the
 * page fixes no format): the two GEMMs fed by a LayerNorm in every layer (q,
 * k, v and fc1) take e4m3 operands, scaled per weight output channel and per
 * activation row so that each row's largest magnitude maps to 448:
 *   s_w[n] = fp32(max_k |w[n][k]|) / 448,  w8 = e4m3(w / s_w[n])
 *   s_a[m] = fp32(max_k |y[m][k]|) / 448,  a8 = e4m3(y / s_a[m])
 *   out[m][n] = (sum_k a8 w8) * s_a[m] * s_w[n] + b[n]
 * e4m3: 1 sign, 4 exponent (bias 7) and 3 mantissa bits, largest finite
 * 448, smallest step 2^-9; conversion rounds to nearest, ties to even, and
 * saturates at +-448 (fp32 arithmetic for the scales and the divisions; a
 * zero row or channel has scale 0 and operands 0). */

/* fp32 -> the nearest e4m3 value (ties to even), saturating at +-448. */
float oracle_e4m3(float x)
{
    if (x != x) return x;
    const float a = fabsf(x);
    float r;
    if (a >= 448.0f) {
        r = 448.0f;
    } else {
        int e;
        frexpf(a, &e);  /* a = f * 2^e, f in [0.5, 1): the leading bit is 2^(e-1) */
        int lead = e - 1;
        if (lead < -6) lead = -6;  /* below the normal range the step stays 2^-9 */
        const float step = ldexpf(1.0f, lead - 3);
        r = rintf(a / step) * step;  /* exact: a / step and the product are powers-of-two scalings */
        if (r > 448.0f) r = 448.0f;
    }
    return x < 0.0f ? -r : r;
}

/* Quantise w [rows][cols] (bf16 bits) per row: q receives e4m3 values as
 * bf16 bits (every e4m3 value is a bf16 value), scales s[row]. */
void oracle_quant_e4m3_rows(const uint16_t *w, int rows, int cols, uint16_t *q, float *scales)
{
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; r++) {
        const uint16_t *x = w + (size_t)r * cols;
        float amax = 0.0f;
        for (int k = 0; k < cols; k++) {
            const float a = fabsf(bff(x[k]));
            if (a > amax) amax = a;
        }
        const float s = amax / 448.0f;
        scales[r] = s;
        for (int k = 0; k < cols; k++)
            q[(size_t)r * cols + k] = s > 0.0f ? bf16_rne(oracle_e4m3(bff(x[k]) / s)) : 0;
    }
}

/* Quantise activation rows y [M][K] in place to e4m3 values, scales s[M]. */
static void quant_e4m3_act(float *y, int64_t M, int K, float *s)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        float *r = y + m * K;
        float amax = 0.0f;
        for (int k = 0; k < K; k++) {
            const float a = fabsf(r[k]);
            if (a > amax) amax = a;
        }
        const float sc = amax / 448.0f;
        s[m] = sc;
        for (int k = 0; k < K; k++) r[k] = sc > 0.0f ? oracle_e4m3(r[k] / sc) : 0.0f;
    }
}

/* The blob's [out][in] matrix at p, quantised when bits == 4, transposed. */
static uint16_t *take_linear(const uint16_t *p, int out, int in, int bits)
{
    if (bits != 4) return transpose_bf16(p, out, in);
    uint16_t *q = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)out * in);
    oracle_quant_rtn4(p, out, in, q, NULL, NULL);
    uint16_t *t = transpose_bf16(q, out, in);
    free(q);
    return t;
}

/* The blob's [out][in] matrix at p as e4m3 values per output channel,
 * transposed; *scales receives s_w [out] (malloc'd). */
static uint16_t *take_linear_e4m3(const uint16_t *p, int out, int in, float **scales)
{
    uint16_t *q = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)out * in);
    *scales = (float *)malloc(sizeof(float) * out);
    oracle_quant_e4m3_rows(p, out, in, q, *scales);
    uint16_t *t = transpose_bf16(q, out, in);
    free(q);
    return t;
}

/* ------------------------------------------------ NVFP4 GEMM operands
 *
 * Page "Ossicle-4B", "Quantized: NVFP4 and INT4 in vLLM": the nvfp4 build
 * quantises the weights and the activations of the audio encoder to NVFP4
 * with NVIDIA ModelOpt and runs on Blackwell's native FP4 kernels.  Reading
 * (the page names the format, no more): NVFP4 as ModelOpt defines it.
 * Elements are E2M1 (1 sign, 2 exponent and 1 mantissa bit: 0, 0.5, 1, 1.5,
 * 2, 3, 4, 6 and their negatives); each block of 16 consecutive elements
 * along the contraction shares a positive E4M3 scale; one fp32 scale g
 * covers a whole tensor, so that the block scales use E4M3's range:
 *   g = fp32(amax) / 2688          (2688 = 6 x 448)
 *   s_b = e4m3(fp32(amax_b) / (g * 6))
 *   q = e2m1(x / (s_b * g))        (0 when s_b = 0; ties to even, +-6 saturates)
 *   x' = q * s_b * g
 * all in fp32.  Weights: one g per weight matrix.  Activations (the
 * LayerNorm rows that feed q, k, v and fc1, the GEMMs the FP8 reading also
 * takes): one g per row, so that a row's operands never depend on the other
 * rows of a batch.  A GEMM is then
 *   out[m][n] = (sum_k (q_a s_a)[m][k] (q_w s_w)[n][k]) * g_a[m] * g_w + b[n]
 * where every product q s (at most 7 significant bits) is exact in bf16. */

/* fp32 -> the nearest E2M1 value (ties to even), saturating at +-6. */
float oracle_e2m1(float x)
{
    if (x != x) return x;
    static const float grid[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    const float a = fabsf(x);
    float r = 6.0f;
    for (int i = 0; i < 7; i++) {
        const float mid = 0.5f * (grid[i] + grid[i + 1]);  /* exact */
        if (a < mid || (a == mid && (i % 2) == 0)) {  /* grid[i] has an even code when i is even */
            r = grid[i];
            break;
        }
        if (a == mid) {  /* the tie goes up to the even code */
            r = grid[i + 1];
            break;
        }
    }
    return x < 0.0f ? -r : r;
}

/* NVFP4 quantisation of x [rows][cols] (cols a multiple of 16).  With
 * per_row, one g per row (g[rows]), else one g for the whole matrix (g[0]).
 * unit[r][k] receives q * s_b (the operand the tensor cores multiply, before
 * g), codes[r][k] the E2M1 code (sign bit 3, magnitude index 0..7),
 * bscale[r][k / 16] the block scales; codes and bscale may be NULL. */
void oracle_quant_nvfp4(const float *x, int64_t rows, int cols, int per_row, float *unit, float *g,
                        uint8_t *codes, float *bscale)
{
    float gt = 0.0f;
    if (!per_row) {
        float amax = 0.0f;
        for (int64_t i = 0; i < rows * (int64_t)cols; i++) {
            const float a = fabsf(x[i]);
            if (a > amax) amax = a;
        }
        gt = amax / 2688.0f;
        g[0] = gt;
    }
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        const float *xr = x + r * cols;
        float gr = gt;
        if (per_row) {
            float amax = 0.0f;
            for (int k = 0; k < cols; k++) {
                const float a = fabsf(xr[k]);
                if (a > amax) amax = a;
            }
            gr = amax / 2688.0f;
            g[r] = gr;
        }
        for (int b0 = 0; b0 < cols; b0 += 16) {
            float bmax = 0.0f;
            for (int k = b0; k < b0 + 16; k++) {
                const float a = fabsf(xr[k]);
                if (a > bmax) bmax = a;
            }
            const float sb = gr > 0.0f ? oracle_e4m3(bmax / (gr * 6.0f)) : 0.0f;
            if (bscale) bscale[r * (cols / 16) + b0 / 16] = sb;
            const float sg = sb * gr;
            for (int k = b0; k < b0 + 16; k++) {
                const float q = sb > 0.0f ? oracle_e2m1(xr[k] / sg) : 0.0f;
                unit[r * cols + k] = q * sb;
                if (codes) {
                    static const float grid[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
                    int idx = 0;
                    while (grid[idx] != fabsf(q)) idx++;
                    codes[r * cols + k] = (uint8_t)(idx | (q < 0.0f || (q == 0.0f && signbit(q)) ? 8 : 0));
                }
            }
        }
    }
}

/* The blob's [out][in] matrix at p as NVFP4 units q * s_b (bf16 bits, exact),
 * transposed; *g receives the matrix's g repeated out times (malloc'd), the
 * per-column factor of linear_e4m3. */
static uint16_t *take_linear_nvfp4(const uint16_t *p, int out, int in, float **g)
{
    float *x = (float *)malloc(sizeof(float) * (size_t)out * in);
    float *u = (float *)malloc(sizeof(float) * (size_t)out * in);
    for (size_t i = 0; i < (size_t)out * in; i++) x[i] = bff(p[i]);
    float gw = 0.0f;
    oracle_quant_nvfp4(x, out, in, 0, u, &gw, NULL, NULL);
    uint16_t *q = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)out * in);
    for (size_t i = 0; i < (size_t)out * in; i++) q[i] = bf16_rne(u[i]);
    uint16_t *t = transpose_bf16(q, out, in);
    *g = (float *)malloc(sizeof(float) * out);
    for (int n = 0; n < out; n++) (*g)[n] = gw;
    free(x); free(u); free(q);
    return t;
}

/* Activation rows y [M][K] in place -> NVFP4 units q * s_b, g[M] per row. */
static void quant_nvfp4_act(float *y, int64_t M, int K, float *g)
{
    float *u = (float *)malloc(sizeof(float) * (size_t)M * K);
    oracle_quant_nvfp4(y, M, K, 1, u, g, NULL, NULL);
    memcpy(y, u, sizeof(float) * (size_t)M * K);
    free(u);
}

/* weight_bits value of the NVFP4 model (oracle_model_create_nvfp4) */
#define NVFP4_BITS 0x4f4

/* Walks the blob in its documented order (conv1, conv2, conv3, conv_out,
 * layers, ln_post, proj1, proj2, adapter gate/up/down; each weight followed
 * by its bias, none for conv_out).  weight_bits 4 gives the 4-bit model of
 * the quantisation section above (its linear layers' weights w'), 8 the FP8
 * model (q, k, v and fc1 on e4m3 operands), any other value the bf16 model. */
oracle_model *oracle_model_create_bits(const uint16_t *blob, int n_layers, int weight_bits)
{
    oracle_model *m = (oracle_model *)calloc(1, sizeof(oracle_model));
    const uint16_t *p = blob;
    m->n_layers = n_layers;
    m->fp8 = weight_bits == 8;
    m->nvfp4 = weight_bits == NVFP4_BITS;
    int cin[3] = {1, C_STEM, C_STEM};
    for (int c = 0; c < 3; c++) {
        m->conv_in[c] = cin[c];
        const uint16_t *w = p;
        p += (size_t)C_STEM * cin[c] * 9;
        m->conv_b[c] = p;
        p += C_STEM;
        float *t = (float *)malloc(sizeof(float) * (size_t)cin[c] * 9 * C_STEM);
        for (int o = 0; o < C_STEM; o++)
            for (int i = 0; i < cin[c]; i++)
                for (int kk = 0; kk < 9; kk++)
                    t[((size_t)i * 9 + kk) * C_STEM + o] = bff(w[((size_t)o * cin[c] + i) * 9 + kk]);
        m->conv_w_t[c] = t;
    }
    m->conv_out_t = transpose_bf16(p, D, C_STEM * F_STEM);
    p += (size_t)D * C_STEM * F_STEM;
    m->layers = (layer_w *)calloc(n_layers > 0 ? n_layers : 1, sizeof(layer_w));
    for (int l = 0; l < n_layers; l++) {
        layer_w *L = &m->layers[l];
        L->ln1_g = p; p += D;
        L->ln1_b = p; p += D;
        if (weight_bits == 8) L->wq_t = take_linear_e4m3(p, D, D, &L->sq);
        else if (weight_bits == NVFP4_BITS) L->wq_t = take_linear_nvfp4(p, D, D, &L->sq);
        else L->wq_t = take_linear(p, D, D, weight_bits);
        p += (size_t)D * D;
        L->bq = p; p += D;
        if (weight_bits == 8) L->wk_t = take_linear_e4m3(p, D, D, &L->sk);
        else if (weight_bits == NVFP4_BITS) L->wk_t = take_linear_nvfp4(p, D, D, &L->sk);
        else L->wk_t = take_linear(p, D, D, weight_bits);
        p += (size_t)D * D;
        L->bk = p; p += D;
        if (weight_bits == 8) L->wv_t = take_linear_e4m3(p, D, D, &L->sv);
        else if (weight_bits == NVFP4_BITS) L->wv_t = take_linear_nvfp4(p, D, D, &L->sv);
        else L->wv_t = take_linear(p, D, D, weight_bits);
        p += (size_t)D * D;
        L->bv = p; p += D;
        L->wo_t = take_linear(p, D, D, weight_bits); p += (size_t)D * D;
        L->bo = p; p += D;
        L->ln2_g = p; p += D;
        L->ln2_b = p; p += D;
        if (weight_bits == 8) L->w1_t = take_linear_e4m3(p, D_FFN, D, &L->s1);
        else if (weight_bits == NVFP4_BITS) L->w1_t = take_linear_nvfp4(p, D_FFN, D, &L->s1);
        else L->w1_t = take_linear(p, D_FFN, D, weight_bits);
        p += (size_t)D_FFN * D;
        L->b1 = p; p += D_FFN;
        L->w2_t = take_linear(p, D, D_FFN, weight_bits); p += (size_t)D * D_FFN;
        L->b2 = p; p += D;
    }
    m->lnp_g = p; p += D;
    m->lnp_b = p; p += D;
    m->wp1_t = take_linear(p, D, D, weight_bits); p += (size_t)D * D;
    m->bp1 = p; p += D;
    m->wp2_t = take_linear(p, D_OUT, D, weight_bits); p += (size_t)D_OUT * D;
    m->bp2 = p; p += D_OUT;
    m->wg_t = take_linear(p, D_ADP, D_OUT, weight_bits); p += (size_t)D_ADP * D_OUT;
    m->bg = p; p += D_ADP;
    m->wu_t = take_linear(p, D_ADP, D_OUT, weight_bits); p += (size_t)D_ADP * D_OUT;
    m->bu = p; p += D_ADP;
    m->wd_t = take_linear(p, D_OUT, D_ADP, weight_bits); p += (size_t)D_OUT * D_ADP;
    m->bd = p; p += D_OUT;
    return m;
}

oracle_model *oracle_model_create_nvfp4(const uint16_t *blob, int n_layers)
{
    return oracle_model_create_bits(blob, n_layers, NVFP4_BITS);
}

oracle_model *oracle_model_create(const uint16_t *blob, int n_layers)
{
    return oracle_model_create_bits(blob, n_layers, 16);
}

/* Number of bf16 elements the blob holds for n_layers layers. */
int64_t oracle_weight_count(int n_layers)
{
    int64_t n = 0;
    n += (int64_t)C_STEM * 9 + C_STEM;
    n += 2 * ((int64_t)C_STEM * C_STEM * 9 + C_STEM);
    n += (int64_t)D * C_STEM * F_STEM;
    int64_t per_layer = 4 * (int64_t)D + 4 * ((int64_t)D * D + D) +
                        ((int64_t)D_FFN * D + D_FFN) + ((int64_t)D * D_FFN + D);
    n += per_layer * n_layers;
    n += 2 * (int64_t)D + ((int64_t)D * D + D) + ((int64_t)D_OUT * D + D_OUT);
    n += 2 * ((int64_t)D_ADP * D_OUT + D_ADP) + ((int64_t)D_OUT * D_ADP + D_OUT);
    return n;
}

void oracle_model_destroy(oracle_model *m)
{
    if (!m) return;
    for (int c = 0; c < 3; c++) free(m->conv_w_t[c]);
    free(m->conv_out_t);
    for (int l = 0; l < m->n_layers; l++) {
        layer_w *L = &m->layers[l];
        free(L->wq_t); free(L->wk_t); free(L->wv_t); free(L->wo_t);
        free(L->w1_t); free(L->w2_t);
        free(L->sq); free(L->sk); free(L->sv); free(L->s1);
    }
    free(m->layers);
    free(m->wp1_t); free(m->wp2_t); free(m->wg_t); free(m->wu_t); free(m->wd_t);
    free(m);
}

/* ---------------------------------------------------------------- primitives */

static double gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }
static double silu(double x) { return x / (1.0 + exp(-x)); }

/* y[m][n] = b[n] + sum_k x[m][k] w[n][k], with w given transposed [K][N].
 * Each output sums over k in order, in fp64. */
static void linear(const float *x, int64_t M, int K, const uint16_t *wt, const uint16_t *bias,
                   int N, float *y)
{
#pragma omp parallel
    {
        double *acc = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t m = 0; m < M; m++) {
            for (int n = 0; n < N; n++) acc[n] = 0.0;
            const float *xr = x + m * K;
            for (int k = 0; k < K; k++) {
                double a = xr[k];
                const uint16_t *w = wt + (size_t)k * N;
                for (int n = 0; n < N; n++) acc[n] += a * (double)bff(w[n]);
            }
            for (int n = 0; n < N; n++)
                y[m * N + n] = (float)(acc[n] + (bias ? bf(bias[n]) : 0.0));
        }
        free(acc);
    }
}

/* The FP8 GEMM: y[m][n] = (sum_k x8[m][k] w8[n][k]) * sa[m] * sw[n] + b[n],
 * x8 and w8 e4m3 values (w8 given transposed [K][N] as bf16 bits), the sum
 * in fp64 over k in order. */
static void linear_e4m3(const float *x8, int64_t M, int K, const uint16_t *w8t, const float *sa, const float *sw,
                        const uint16_t *bias, int N, float *y)
{
#pragma omp parallel
    {
        double *acc = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t m = 0; m < M; m++) {
            for (int n = 0; n < N; n++) acc[n] = 0.0;
            const float *xr = x8 + m * K;
            for (int k = 0; k < K; k++) {
                double a = xr[k];
                const uint16_t *w = w8t + (size_t)k * N;
                for (int n = 0; n < N; n++) acc[n] += a * (double)bff(w[n]);
            }
            for (int n = 0; n < N; n++) y[m * N + n] = (float)(acc[n] * sa[m] * sw[n] + bf(bias[n]));
        }
        free(acc);
    }
}

/* LayerNorm over the last dimension (biased variance, eps 1e-5). */
static void layernorm(const float *x, int64_t M, int N, const uint16_t *g, const uint16_t *b,
                      float *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        const float *r = x + m * N;
        double mean = 0.0, var = 0.0;
        for (int n = 0; n < N; n++) mean += r[n];
        mean /= N;
        for (int n = 0; n < N; n++) var += (r[n] - mean) * (r[n] - mean);
        var /= N;
        double rstd = 1.0 / sqrt(var + LN_EPS);
        for (int n = 0; n < N; n++) y[m * N + n] = (float)((r[n] - mean) * rstd * bf(g[n]) + bf(b[n]));
    }
}

/* Conv2D, kernel 3x3, stride 2, padding 1, then + bias and GELU.
 * in [Cin][H][W], weights transposed [Cin][3][3][Cout], out [Cout][Ho][Wo].
 * H is the mel (frequency) axis and W the time axis. */
static void conv3x3s2_gelu(const float *in, int Cin, int H, int W, const float *wt,
                           const uint16_t *bias, int Cout, float *out)
{
    int Ho = (H + 2 - 3) / 2 + 1, Wo = (W + 2 - 3) / 2 + 1;
#pragma omp parallel
    {
        double *acc = (double *)malloc(sizeof(double) * Cout);
#pragma omp for collapse(2) schedule(static)
        for (int fo = 0; fo < Ho; fo++)
            for (int to = 0; to < Wo; to++) {
                for (int o = 0; o < Cout; o++) acc[o] = 0.0;
                for (int i = 0; i < Cin; i++)
                    for (int kf = 0; kf < 3; kf++) {
                        int fi = 2 * fo + kf - 1;
                        if (fi < 0 || fi >= H) continue;
                        for (int kt = 0; kt < 3; kt++) {
                            int ti = 2 * to + kt - 1;
                            if (ti < 0 || ti >= W) continue;
                            double a = in[((size_t)i * H + fi) * W + ti];
                            const float *w = wt + ((size_t)i * 9 + kf * 3 + kt) * Cout;
                            for (int o = 0; o < Cout; o++) acc[o] += a * (double)w[o];
                        }
                    }
                for (int o = 0; o < Cout; o++)
                    out[((size_t)o * Ho + fo) * Wo + to] = (float)gelu(acc[o] + bf(bias[o]));
            }
        free(acc);
    }
}

/* Sinusoidal position p, channel c of 1280: channels 0..639 are
 * sin(p * inv_i), channels 640..1279 are cos(p * inv_i), with
 * inv_i = exp(-i * ln(10000) / 639). */
double oracle_position(int p, int c)
{
    int half = D / 2;
    int i = c < half ? c : c - half;
    double inv = exp(-(double)i * log(10000.0) / (half - 1));
    return c < half ? sin(p * inv) : cos(p * inv);
}

/* Stem of one chunk: the normalised mel of Fc <= 800 frames ([Fc][128],
 * frame-major) is zero-padded to 800 frames, run through conv1..conv3
 * (GELU after each) over the (freq=128, time=800) plane, flattened per output
 * time step as index c*16+f, projected by conv_out (no bias), and the chunk-
 * local sinusoidal position is added.  Writes the first ceil(Fc/8) rows of
 * x_out [Tc][1280]; returns Tc. */
int oracle_stem_chunk(const oracle_model *m, const float *mel_norm, int Fc, float *x_out)
{
    if (Fc <= 0) return 0;
    int Tc = (int)oracle_chunk_tokens(Fc);
    const int H0 = N_MELS, W0 = CHUNK_FRAMES;
    float *img = (float *)calloc((size_t)H0 * W0, sizeof(float));
    for (int t = 0; t < Fc; t++)
        for (int f = 0; f < N_MELS; f++) img[(size_t)f * W0 + t] = mel_norm[(size_t)t * N_MELS + f];
    int H1 = 64, W1 = 400, H2 = 32, W2 = 200, H3 = 16, W3 = 100;
    float *o1 = (float *)malloc(sizeof(float) * (size_t)C_STEM * H1 * W1);
    float *o2 = (float *)malloc(sizeof(float) * (size_t)C_STEM * H2 * W2);
    float *o3 = (float *)malloc(sizeof(float) * (size_t)C_STEM * H3 * W3);
    conv3x3s2_gelu(img, 1, H0, W0, m->conv_w_t[0], m->conv_b[0], C_STEM, o1);
    conv3x3s2_gelu(o1, C_STEM, H1, W1, m->conv_w_t[1], m->conv_b[1], C_STEM, o2);
    conv3x3s2_gelu(o2, C_STEM, H2, W2, m->conv_w_t[2], m->conv_b[2], C_STEM, o3);
    float *flat = (float *)malloc(sizeof(float) * (size_t)Tc * C_STEM * F_STEM);
    for (int t = 0; t < Tc; t++)
        for (int c = 0; c < C_STEM; c++)
            for (int f = 0; f < F_STEM; f++)
                flat[(size_t)t * C_STEM * F_STEM + c * F_STEM + f] = o3[((size_t)c * H3 + f) * W3 + t];
    linear(flat, Tc, C_STEM * F_STEM, m->conv_out_t, NULL, D, x_out);
    for (int t = 0; t < Tc; t++)
        for (int c = 0; c < D; c++)
            x_out[(size_t)t * D + c] = (float)((double)x_out[(size_t)t * D + c] + oracle_position(t, c));
    free(img); free(o1); free(o2); free(o3); free(flat);
    return Tc;
}

/* Attention inside windows.  win[w]..win[w+1] are the token ranges of the
 * windows.  Block-diagonal form: every query attends only the keys of its own
 * window.  scores = q.k / sqrt(64), softmax in fp64. */
static void attention_blockdiag(const float *q, const float *k, const float *v, const int *win,
                                int n_win, float *o)
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int w = 0; w < n_win; w++)
        for (int h = 0; h < N_HEADS; h++) {
            int s = win[w], e = win[w + 1], n = e - s;
            if (n <= 0) continue;
            double *sc = (double *)malloc(sizeof(double) * n);
            for (int i = s; i < e; i++) {
                double mx = -INFINITY;
                for (int j = s; j < e; j++) {
                    double d = 0.0;
                    for (int c = 0; c < HEAD_DIM; c++)
                        d += (double)q[(size_t)i * D + h * HEAD_DIM + c] * k[(size_t)j * D + h * HEAD_DIM + c];
                    sc[j - s] = d / sqrt((double)HEAD_DIM);
                    mx = sc[j - s] > mx ? sc[j - s] : mx;
                }
                double sum = 0.0;
                for (int j = 0; j < n; j++) { sc[j] = exp(sc[j] - mx); sum += sc[j]; }
                for (int c = 0; c < HEAD_DIM; c++) {
                    double acc = 0.0;
                    for (int j = s; j < e; j++) acc += sc[j - s] * v[(size_t)j * D + h * HEAD_DIM + c];
                    o[(size_t)i * D + h * HEAD_DIM + c] = (float)(acc / sum);
                }
            }
            free(sc);
        }
}

/* The same attention written as full T x T attention with a mask that is
 * -inf wherever query and key lie in different windows. */
static void attention_full_masked(const float *q, const float *k, const float *v, const int *win,
                                  int n_win, int T, float *o)
{
    int *wid = (int *)malloc(sizeof(int) * (T > 0 ? T : 1));
    for (int w = 0; w < n_win; w++)
        for (int t = win[w]; t < win[w + 1]; t++) wid[t] = w;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int i = 0; i < T; i++)
        for (int h = 0; h < N_HEADS; h++) {
            double *sc = (double *)malloc(sizeof(double) * T);
            double mx = -INFINITY;
            for (int j = 0; j < T; j++) {
                double d = 0.0;
                for (int c = 0; c < HEAD_DIM; c++)
                    d += (double)q[(size_t)i * D + h * HEAD_DIM + c] * k[(size_t)j * D + h * HEAD_DIM + c];
                double mask = wid[i] == wid[j] ? 0.0 : -INFINITY;
                sc[j] = d / sqrt((double)HEAD_DIM) + mask;
                mx = sc[j] > mx ? sc[j] : mx;
            }
            double sum = 0.0;
            for (int j = 0; j < T; j++) { sc[j] = exp(sc[j] - mx); sum += sc[j]; }
            for (int c = 0; c < HEAD_DIM; c++) {
                double acc = 0.0;
                for (int j = 0; j < T; j++) acc += sc[j] * v[(size_t)j * D + h * HEAD_DIM + c];
                o[(size_t)i * D + h * HEAD_DIM + c] = (float)(acc / sum);
            }
            free(sc);
        }
    free(wid);
}

/* Pre-LN Transformer layers l0..l1-1 over x [T][1280] in place:
 *   x += o(attn(LN1 x)); x += fc2(GELU(fc1(LN2 x))). */
int oracle_layers(const oracle_model *m, float *x, int T, const int *win, int n_win, int l0,
                  int l1, int attn_full)
{
    if (T <= 0) return 0;
    size_t td = (size_t)T * D;
    float *h = (float *)malloc(sizeof(float) * td);
    float *q = (float *)malloc(sizeof(float) * td);
    float *k = (float *)malloc(sizeof(float) * td);
    float *v = (float *)malloc(sizeof(float) * td);
    float *a = (float *)malloc(sizeof(float) * td);
    float *f = (float *)malloc(sizeof(float) * (size_t)T * D_FFN);
    float *sa = (float *)malloc(sizeof(float) * (size_t)T);
    for (int l = l0; l < l1; l++) {
        const layer_w *L = &m->layers[l];
        layernorm(x, T, D, L->ln1_g, L->ln1_b, h);
        if (m->nvfp4) {
            quant_nvfp4_act(h, T, D, sa);
            linear_e4m3(h, T, D, L->wq_t, sa, L->sq, L->bq, D, q);
            linear_e4m3(h, T, D, L->wk_t, sa, L->sk, L->bk, D, k);
            linear_e4m3(h, T, D, L->wv_t, sa, L->sv, L->bv, D, v);
        } else if (m->fp8) {
            quant_e4m3_act(h, T, D, sa);
            linear_e4m3(h, T, D, L->wq_t, sa, L->sq, L->bq, D, q);
            linear_e4m3(h, T, D, L->wk_t, sa, L->sk, L->bk, D, k);
            linear_e4m3(h, T, D, L->wv_t, sa, L->sv, L->bv, D, v);
        } else {
            linear(h, T, D, L->wq_t, L->bq, D, q);
            linear(h, T, D, L->wk_t, L->bk, D, k);
            linear(h, T, D, L->wv_t, L->bv, D, v);
        }
        if (attn_full)
            attention_full_masked(q, k, v, win, n_win, T, a);
        else
            attention_blockdiag(q, k, v, win, n_win, a);
        linear(a, T, D, L->wo_t, L->bo, D, h);
        for (size_t i = 0; i < td; i++) x[i] = (float)((double)x[i] + h[i]);
        layernorm(x, T, D, L->ln2_g, L->ln2_b, h);
        if (m->nvfp4) {
            quant_nvfp4_act(h, T, D, sa);
            linear_e4m3(h, T, D, L->w1_t, sa, L->s1, L->b1, D_FFN, f);
        } else if (m->fp8) {
            quant_e4m3_act(h, T, D, sa);
            linear_e4m3(h, T, D, L->w1_t, sa, L->s1, L->b1, D_FFN, f);
        } else {
            linear(h, T, D, L->w1_t, L->b1, D_FFN, f);
        }
        for (size_t i = 0; i < (size_t)T * D_FFN; i++) f[i] = (float)gelu(f[i]);
        linear(f, T, D_FFN, L->w2_t, L->b2, D, h);
        for (size_t i = 0; i < td; i++) x[i] = (float)((double)x[i] + h[i]);
    }
    free(h); free(q); free(k); free(v); free(a); free(f); free(sa);
    return 0;
}

/* Encoder head: ln_post -> proj1 -> GELU -> proj2.  x [T][1280] -> out [T][2048]. */
int oracle_head(const oracle_model *m, const float *x, int T, float *out)
{
    if (T <= 0) return 0;
    float *h = (float *)malloc(sizeof(float) * (size_t)T * D);
    float *p = (float *)malloc(sizeof(float) * (size_t)T * D);
    layernorm(x, T, D, m->lnp_g, m->lnp_b, h);
    linear(h, T, D, m->wp1_t, m->bp1, D, p);
    for (size_t i = 0; i < (size_t)T * D; i++) p[i] = (float)gelu(p[i]);
    linear(p, T, D, m->wp2_t, m->bp2, D_OUT, out);
    free(h); free(p);
    return 0;
}

/* SwiGLU adapter: y = down(SiLU(gate(h)) * up(h)).  h, y [T][2048]. */
int oracle_adapter(const oracle_model *m, const float *h, int T, float *y)
{
    if (T <= 0) return 0;
    float *g = (float *)malloc(sizeof(float) * (size_t)T * D_ADP);
    float *u = (float *)malloc(sizeof(float) * (size_t)T * D_ADP);
    linear(h, T, D_OUT, m->wg_t, m->bg, D_ADP, g);
    linear(h, T, D_OUT, m->wu_t, m->bu, D_ADP, u);
    for (size_t i = 0; i < (size_t)T * D_ADP; i++) g[i] = (float)(silu(g[i]) * (double)u[i]);
    linear(g, T, D_ADP, m->wd_t, m->bd, D_OUT, y);
    free(g); free(u);
    return 0;
}

/* Encode the 800-frame chunks [c0, c1) of one clip.  Each chunk is one
 * attention window.  gmax is the clip's log-mel maximum; pass NaN to compute
 * it over the whole clip.  out [T][2048] receives the rows of those chunks in
 * order (T = their token count, returned).  Optional dumps (NULL to skip):
 * stem [T][1280] after conv_out + positions, enc [T][1280] after the last
 * layer, head [T][2048] after proj2.  attn_full selects the full masked form
 * of the attention instead of the block-diagonal one. */
int64_t oracle_encode_chunks(const oracle_model *m, const float *pcm, int64_t n, int64_t c0,
                             int64_t c1, float gmax, int attn_full, float *out, float *dump_stem,
                             float *dump_enc, float *dump_head)
{
    int64_t F = oracle_num_frames(n);
    int64_t nc = oracle_num_chunks(n);
    if (c0 < 0) c0 = 0;
    if (c1 > nc) c1 = nc;
    if (c1 <= c0) return 0;
    if (isnan(gmax)) gmax = oracle_clip_log_max(pcm, n);
    int n_win = (int)(c1 - c0);
    int *win = (int *)malloc(sizeof(int) * (n_win + 1));
    int T = 0;
    win[0] = 0;
    for (int64_t c = c0; c < c1; c++) {
        int64_t fc = F - c * CHUNK_FRAMES < CHUNK_FRAMES ? F - c * CHUNK_FRAMES : CHUNK_FRAMES;
        T += (int)oracle_chunk_tokens(fc);
        win[c - c0 + 1] = T;
    }
    float *x = (float *)malloc(sizeof(float) * (size_t)T * D);
    float *mel = (float *)malloc(sizeof(float) * CHUNK_FRAMES * N_MELS);
    for (int64_t c = c0; c < c1; c++) {
        int64_t f0 = c * CHUNK_FRAMES;
        int64_t fc = F - f0 < CHUNK_FRAMES ? F - f0 : CHUNK_FRAMES;
        oracle_logmel_raw(pcm, n, f0, f0 + fc, mel);
        oracle_normalize(mel, fc * N_MELS, gmax);
        oracle_stem_chunk(m, mel, (int)fc, x + (size_t)win[c - c0] * D);
    }
    if (dump_stem) memcpy(dump_stem, x, sizeof(float) * (size_t)T * D);
    oracle_layers(m, x, T, win, n_win, 0, m->n_layers, attn_full);
    if (dump_enc) memcpy(dump_enc, x, sizeof(float) * (size_t)T * D);
    float *h = (float *)malloc(sizeof(float) * (size_t)T * D_OUT);
    oracle_head(m, x, T, h);
    if (dump_head) memcpy(dump_head, h, sizeof(float) * (size_t)T * D_OUT);
    oracle_adapter(m, h, T, out);
    free(h); free(x); free(mel); free(win);
    return T;
}
