/*
 * moss_enc: audio-encoder forward of the MOSS-Audio / MOSS-Transcribe family
 * (the Qwen3-Omni AuT tower) for NVIDIA B200 (sm_100a).
 *
 * The method (page "MOSS-Transcribe-preview-2B - GGUF", "Architecture" table):
 * 16 kHz mono PCM -> Whisper-style 128-bin log-mel (n_fft 400, hop 160) ->
 * 3 x Conv2D stride 2 (1->480->480->480) -> conv_out (480*16 = 7680 -> 1280,
 * no bias) + sinusoidal positions -> 32 pre-LN Transformer layers (d 1280,
 * 20 heads x 64, FFN 5120) with windowed (block-diagonal) attention ->
 * ln_post -> proj1 (1280->1280) -> GELU -> proj2 (1280->2048) -> SwiGLU
 * adapter (2048->8192->2048).  The caller gets 12.5 rows per second of audio
 * (page "Ossicle-4B", "Model Overview").
 *
 * Conventions for every call:
 *  - Pointers documented as "device" must be device memory of the handle's
 *    device; "host" pointers are ordinary (preferably pinned) host memory.
 *  - Calls that take a handle enqueue their work on the handle's stream and
 *    return without waiting, except where a call says it synchronises.  The
 *    caller keeps device inputs alive and unmodified until the work is done.
 *  - No call allocates device memory after moss_enc_create; a request larger
 *    than the capacity fixed at create time returns MOSS_ENC_ERR_CAPACITY.
 *  - No C++ exception crosses this interface.  A handle is used by one host
 *    thread at a time.
 *  - Errors found on the device (a bounded wait that timed out) are reported
 *    by moss_enc_synchronize.
 */
#ifndef MOSS_ENC_H
#define MOSS_ENC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOSS_ENC_OK = 0,
    MOSS_ENC_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad size or range */
    MOSS_ENC_ERR_CAPACITY = 2,       /* request exceeds the capacity set at create */
    MOSS_ENC_ERR_OOM = 3,            /* device allocation failed inside create */
    MOSS_ENC_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
    MOSS_ENC_ERR_DEVICE_TIMEOUT = 5  /* a kernel's bounded wait gave up */
} moss_enc_status;

typedef struct moss_enc moss_enc; /* opaque; owned by the library */

/* Output element type of the embedding rows. */
enum { MOSS_ENC_OUT_F32 = 0, MOSS_ENC_OUT_BF16 = 1 };

/* Forward stages, for moss_enc_forward_stage (boundary checks). */
enum {
    MOSS_ENC_STAGE_STEM = 0,    /* after conv_out + positions: fp32 [T][1280] */
    MOSS_ENC_STAGE_LAYERS = 1,  /* after the last layer, before ln_post: fp32 [T][1280] */
    MOSS_ENC_STAGE_HEAD = 2,    /* after proj2: fp32 [T][2048] */
    MOSS_ENC_STAGE_ADAPTER = 3  /* final rows: out_dtype [T][2048] (same as moss_enc_forward) */
};

typedef struct {
    int n_layers;          /* 1..32 encoder layers held by the weight blob */
    int64_t max_samples;   /* capacity: sum over clips of encoded samples per call */
    int max_clips;         /* capacity: clips per call */
    int out_dtype;         /* MOSS_ENC_OUT_F32 or MOSS_ENC_OUT_BF16 */
    int weight_bits;       /* 16 (or 0): bf16 weights; 4: the linear layers of the
                              encoder layers, head and adapter are kept as 4-bit
                              codes (see MOSS_ENC_WEIGHTS_4BIT) */
    int fp8;               /* 1: the q/k/v and fc1 GEMMs of every layer take e4m3
                              operands (see MOSS_ENC_FP8); 0: bf16.  Not with
                              weight_bits = 4. */
    int nvfp4;             /* 1: the q/k/v and fc1 GEMMs of every layer take NVFP4
                              operands (see MOSS_ENC_NVFP4); 0: bf16.  Not with
                              fp8 = 1 or weight_bits = 4. */
} moss_enc_config;

/* FP8 GEMMs (page "Ossicle-4B", "Quantized: NVFP4 and INT4 in vLLM": the
 * low-precision builds quantise the audio encoder's weights and activations
 * for Blackwell's low-precision tensor cores).  With cfg.fp8 = 1 the two
 * GEMMs of every layer that a LayerNorm feeds (q/k/v and fc1) multiply e4m3
 * operands on the tensor cores (kind::f8f6f4, fp32 accumulation):
 *   weights, per output channel n:  s_w[n] = max_k |w[n][k]| / 448,
 *                                   w8 = e4m3(w / s_w[n])   (at create)
 *   LayerNorm rows, per row m:      s_a[m] = max_k |y[m][k]| / 448,
 *                                   a8 = e4m3(y / s_a[m])   (the LayerNorm
 *                                   kernel writes a8 and s_a)
 *   out[m][n] = (sum_k a8 w8) * s_a[m] * s_w[n] + b[n]      (then GELU for fc1)
 * e4m3 rounds to nearest (ties to even) and saturates at +-448; scales and
 * divisions in fp32.  The other GEMMs keep bf16 operands.  The rows then
 * match the FP8 model of the same definition (not the bf16 model). */
#define MOSS_ENC_FP8 1

/* NVFP4 GEMMs (page "Ossicle-4B", section "Quantized: NVFP4 and INT4 in
 * vLLM": an NVFP4 build quantises the audio encoder's weights and
 * activations with NVIDIA ModelOpt and needs Blackwell's native FP4 kernels).
 * With cfg.nvfp4 = 1 the q/k/v and fc1 GEMMs of every layer multiply NVFP4
 * operands on the block-scaled FP4 tensor cores (kind::mxf4nvf4, fp32
 * accumulation).  NVFP4 as ModelOpt defines it: E2M1 elements (0, 0.5, 1,
 * 1.5, 2, 3, 4, 6 and negatives), an E4M3 scale per 16 consecutive k, and one
 * fp32 factor g per tensor:
 *   g = amax / 2688,  s_b = e4m3(amax_b / (g * 6)),  q = e2m1(x / (s_b * g))
 * (fp32 arithmetic, ties to even, saturating; q = 0 when s_b = 0), with one g
 * per weight matrix (q, k, v and fc1 each; at create) and one g per LayerNorm
 * row (the LayerNorm kernel writes the codes, the scales and g, so a row's
 * operands do not depend on the rest of the batch);
 *   out[m][n] = (sum_k q_a s_a q_w s_w) * g_a[m] * g_w + b[n]   (GELU for fc1).
 * The other GEMMs keep bf16 operands.  The rows then match the NVFP4 model of
 * the same definition. */
#define MOSS_ENC_NVFP4 1

/* 4-bit weights (page "Ossicle-4B", "Long Audio", the note under the table:
 * "4-bit weights for ... the audio encoder, round to nearest, groups of 128").
 * With cfg.weight_bits = 4, moss_enc_create quantises the weight matrix of
 * every linear layer of the 32 encoder layers (q, k, v, o, fc1, fc2), of the
 * encoder head (proj1, proj2) and of the adapter (gate, up, down) in groups of
 * 128 consecutive input features of each output row:
 *   s = fp32(max |w|) / 7,  q = clamp(rint(w / s), -8, 7) (0 if s = 0),
 *   w' = bf16(fp32(q * s))   (fp32 arithmetic, ties to even)
 * and keeps only the codes (4 bits) and the scales (fp32 per group); the GEMMs
 * expand them to w' on the fly.  The conv stem (conv1..conv3, conv_out), the
 * biases and the LayerNorm parameters keep their bf16/fp32 values.  Weight
 * memory falls from about 1.4 GB to about 0.4 GB for 32 layers.  Layer taps
 * (moss_enc_set_taps) keep bf16 weights. */
#define MOSS_ENC_WEIGHTS_4BIT 4

/* One clip (or one piece of a clip) to encode.
 *  pcm        device, 16 kHz mono fp32, the WHOLE clip [n_samples].
 *  n_samples  whole-clip length; reflect padding is applied only at sample 0
 *             and at n_samples, so a piece sees its true neighbours.
 *  begin,end  sample range to encode.  begin must be a multiple of 128000
 *             (one 800-frame chunk = 8 s); end must equal n_samples or be a
 *             multiple of 128000.  {0, n_samples} encodes the whole clip.
 *  log_max    device pointer to the clip's log-mel maximum (the Whisper
 *             floor is log_max - 8), or NULL to compute it over the whole
 *             clip [0, n_samples).  Pieces of one long clip pass the value of
 *             moss_enc_log_max so that every piece uses the same floor
 *             (page "Ossicle-4B", "Long Audio": piece log-mel is identical
 *             to the whole clip's). */
typedef struct {
    const float *pcm;
    int64_t n_samples;
    int64_t begin;
    int64_t end;
    const float *log_max;
} moss_enc_clip;

/* ---------------------------------------------------------------- sizes */

/* bf16 elements in the weight blob for n_layers layers.  Blob order
 * (PyTorch layouts, linear [out][in], conv [out][in][k_freq][k_time]):
 *   conv1.w [480][1][3][3], conv1.b [480], conv2.w [480][480][3][3],
 *   conv2.b, conv3.w, conv3.b, conv_out.w [1280][7680] (input index c*16+f,
 *   no bias); per layer: ln1.g, ln1.b [1280], q.w [1280][1280], q.b, k.w,
 *   k.b, v.w, v.b, o.w, o.b, ln2.g, ln2.b, fc1.w [5120][1280], fc1.b [5120],
 *   fc2.w [1280][5120], fc2.b [1280]; then ln_post.g, ln_post.b,
 *   proj1.w [1280][1280], proj1.b, proj2.w [2048][1280], proj2.b [2048],
 *   gate.w [8192][2048], gate.b [8192], up.w [8192][2048], up.b [8192],
 *   down.w [2048][8192], down.b [2048]. */
int64_t moss_enc_weight_count(int n_layers);

/* Mel frames of a clip: n_samples / 160 (Whisper drops the trailing STFT
 * frame; page "MOSS-Transcribe-preview-2B - GGUF", gotcha 2).  Pure. */
int64_t moss_enc_num_frames(int64_t n_samples);

/* Output rows of a whole clip: the sum over 800-frame chunks of
 * ceil(frames_in_chunk / 8) (three stride-2 convs).  Pure.  The rate follows
 * page "Ossicle-4B", "Model Overview" (12.5 audio tokens per second: 100 mel
 * frames per second over an 8x time reduction) and the workload's 8 s chunks
 * (800 frames -> 100 tokens). */
int64_t moss_enc_num_tokens(int64_t n_samples);

/* Output rows of the sample range [begin, end) of a clip of n_samples
 * (same alignment rules as moss_enc_clip).  Returns -1 on a bad range. */
int64_t moss_enc_range_tokens(int64_t n_samples, int64_t begin, int64_t end);

/* ------------------------------------------------------------- lifetime */

/* Create a handle on the current CUDA device.  The handle holds the encoder
 * the page "MOSS-Transcribe-preview-2B - GGUF", "Architecture" table,
 * describes (conv front-end, 32 pre-LN layers, encoder head, SwiGLU adapter);
 * its weights are the blob's, laid out as moss_enc_weight_count says.
 *  weights        bf16 blob (uint16 bit patterns) of moss_enc_weight_count
 *                 (cfg->n_layers) elements; host or device memory as
 *                 weights_on_device says.  The library copies and repacks
 *                 it; the caller may free it when create returns.
 *  bytes          size of the blob in bytes (checked).
 *  stream         cudaStream_t to enqueue on (NULL = legacy default stream).
 *  out            receives the handle.
 * Synchronises.  Allocates the weights and a workspace sized from cfg.
 * Errors: INVALID_ARG (null pointer, n_layers outside 1..32, max_samples or
 * max_clips below 1, unknown out_dtype, wrong byte count), OOM, CUDA (also
 * for a device that is not compute capability 10.x). */
moss_enc_status moss_enc_create(const moss_enc_config *cfg, const void *weights, size_t bytes,
                                int weights_on_device, void *stream, moss_enc **out);

/* Change the stream later calls enqueue on. */
moss_enc_status moss_enc_set_stream(moss_enc *h, void *stream);

/* Wait for the handle's stream; return MOSS_ENC_ERR_DEVICE_TIMEOUT if a kernel
 * reported a timed-out wait since the last call (and clear the flag). */
moss_enc_status moss_enc_synchronize(moss_enc *h);

/* Release a handle: synchronises its stream, then frees the weights, the
 * workspace, the layer taps and any captured forward graph.  NULL is a no-op.
 * The pages describe no teardown of their own; this is the plain counterpart
 * of moss_enc_create. */
void moss_enc_destroy(moss_enc *h);

const char *moss_enc_status_string(moss_enc_status s);

/* Text of the last error on this handle ("" if none). */
const char *moss_enc_last_error(const moss_enc *h);

/* ---------------------------------------------------------------- compute */

/* Whisper log-mel of one clip's range (page "MOSS-Transcribe-preview-2B -
 * GGUF", "Architecture" table, Audio row; gotcha 2): frames t in
 * [begin/160, end/160) (end == n_samples: n_samples/160), each centred on
 * sample 160 t with reflect padding at the clip ends, periodic Hann 400,
 * |rFFT|^2 (201 bins), Slaney mel 128 x 201 over 0-8 kHz, log10(max(., 1e-10)),
 * floor at log_max - 8, then (x + 4) / 4.
 *  mel_out      device fp32 [n_frames][128], frame-major (rows leave by bulk
 *               copies when mel_out is 16-byte aligned, by plain stores
 *               otherwise; the values are the same).
 *  n_frames     host, receives the frame count (may be NULL).
 *  log_max_out  device float receiving the clip's log-mel maximum (may be NULL).
 * The range must hold at most cfg.max_samples samples. */
moss_enc_status moss_enc_logmel(moss_enc *h, const moss_enc_clip *clip, float *mel_out,
                                int64_t *n_frames, float *log_max_out);

/* Whole-clip log-mel maximum only (one pass, nothing else written).
 *  pcm device [n_samples]; out device float.  Any length is accepted. */
moss_enc_status moss_enc_log_max(moss_enc *h, const float *pcm, int64_t n_samples, float *out);

/* Log-mel maximum over the frames of the sample range [begin, end) of a clip
 * (frames t with 160 t in [begin, end); end == n_samples: t < n_samples/160),
 * each frame computed as in the whole clip (reflect padding only at its true
 * ends).  The maximum of the values for ranges that cover a clip is the
 * clip's log_max, so ranks that each encode one range of a long clip agree on
 * the Whisper floor with one max-reduction of a float (page "Ossicle-4B",
 * "Long Audio": pieces use the whole clip's log-mel).
 *  pcm  device [n_samples]; out device float (-inf for an empty range).
 *  begin and end are multiples of 160 (end may also equal n_samples).
 * Nothing else is written. */
moss_enc_status moss_enc_range_log_max(moss_enc *h, const float *pcm, int64_t n_samples, int64_t begin,
                                       int64_t end, float *out);

/* Encode n_clips clips (or pieces) into embedding rows: audio in, one
 * 2048-wide embedding row per 80 ms of audio out, the encoder run once per
 * clip (page "MOSS-Transcribe-preview-2B - GGUF", "Architecture" table, rows
 * Audio, Conv front-end, Audio encoder, Encoder head, Adapter, and
 * "Audio injection"; page "Ossicle-4B", "Long Audio" for pieces of a long
 * clip).
 *  clips        host array [n_clips].
 *  rows_out     device [sum of tokens][2048] of cfg.out_dtype; the rows of
 *               clip i are rows row_offsets[i] .. row_offsets[i+1]-1.
 *  row_offsets  host int64 [n_clips + 1], written before the call returns
 *               (computed on the host, no synchronisation).
 * Each clip is encoded independently: its 800-frame chunks are the conv
 * stem's chunks (zero-padded at the tail) and the attention windows.
 * Errors: INVALID_ARG (null pointer, bad range), CAPACITY (more clips or
 * samples than cfg allows), CUDA. */
moss_enc_status moss_enc_forward(moss_enc *h, const moss_enc_clip *clips, int n_clips,
                                 void *rows_out, int64_t *row_offsets);

/* Like moss_enc_forward but stops after `stage` (MOSS_ENC_STAGE_*) and writes
 * that boundary's rows (fp32 except the final stage) to out. */
moss_enc_status moss_enc_forward_stage(moss_enc *h, const moss_enc_clip *clips, int n_clips,
                                       int stage, void *out, int64_t *row_offsets);

/* ------------------------------------------------------- layer taps */

/* Cross-layer taps (page "MOSS-Audio-4B-Instruct on an RTX 5070", opening
 * paragraph: a DeepStack-inspired cross-layer adapter; page
 * "MOSS-Music-8B-Instruct-GGUF", files section: deepstack injection wiring).
 * A tap takes the residual stream after one encoder layer and runs it through
 * a head + adapter set of its own (ln_post -> proj1 -> GELU -> proj2 ->
 * SwiGLU adapter, the same computation as the encoder's final path), giving
 * [T][2048] rows per tap beside the final rows.  The pages name the idea but
 * not its wiring; this is the plainest reading of it. */
#define MOSS_ENC_MAX_TAPS 8

/* bf16 elements of one tap's head + adapter set, in the order of the tail of
 * the main blob: ln_post.g, ln_post.b [1280], proj1.w [1280][1280], proj1.b,
 * proj2.w [2048][1280], proj2.b [2048], gate.w [8192][2048], gate.b [8192],
 * up.w, up.b, down.w [2048][8192], down.b [2048].  Pure. */
int64_t moss_enc_tap_weight_count(void);

/* Set the taps used by moss_enc_forward_taps (replaces any earlier set).
 *  layers      host int [n_taps]: 0-based encoder layer after which each tap
 *              reads the residual stream (0 <= layer < cfg.n_layers; repeats
 *              allowed).  n_taps 0..MOSS_ENC_MAX_TAPS; 0 removes the taps.
 *  weights     n_taps consecutive sets of moss_enc_tap_weight_count() bf16
 *              elements, host or device memory as weights_on_device says,
 *              copied and repacked (the caller may free it); or NULL to make
 *              every tap use the encoder's own ln_post/proj/adapter weights.
 *  bytes       size of weights in bytes (checked unless weights is NULL).
 * Synchronises the handle's stream and allocates the packed tap weights
 * (about 185 MB per set); forward calls still allocate nothing.
 * Errors: INVALID_ARG (bad list, layer out of range, wrong size), OOM. */
moss_enc_status moss_enc_set_taps(moss_enc *h, const int *layers, int n_taps, const void *weights,
                                  size_t bytes, int weights_on_device);

/* moss_enc_forward plus the tap rows.
 *  tap_rows     host array of n_taps device pointers, tap t's rows
 *               [sum of tokens][2048] of cfg.out_dtype, clip i at rows
 *               row_offsets[i] ..; ignored (may be NULL) with no taps set.
 * Same clips, rows_out, row_offsets and errors as moss_enc_forward. */
moss_enc_status moss_enc_forward_taps(moss_enc *h, const moss_enc_clip *clips, int n_clips,
                                      void *rows_out, void *const *tap_rows, int64_t *row_offsets);

/* End-to-end from host memory: copies each clip's samples host->device,
 * encodes, copies the rows device->host and synchronises.
 *  pcm_host     host array of n_clips pointers to fp32 [n_samples[i]].
 *  n_samples    host [n_clips].
 *  rows_host    host [sum of tokens][2048] of cfg.out_dtype.
 *  row_offsets  host [n_clips + 1].
 * Whole clips only; the sum of n_samples must fit cfg.max_samples. */
moss_enc_status moss_enc_forward_host(moss_enc *h, const float *const *pcm_host,
                                      const int64_t *n_samples, int n_clips, void *rows_host,
                                      int64_t *row_offsets);

/* ------------------------------------------------------- single GEMM */

/* One bf16 GEMM on the tensor cores with a fused epilogue (the kernels every
 * linear layer and conv of the forward use), for tuning and unit tests:
 *   out[M][N] = epi(A[M][K] * B[N][K]^T + bias[N])
 *  A, B       device bf16 (uint16 bits), K-major: A [M][K], B [N][K].
 *  bias       device fp32 [N].
 *  out        device; bf16 [M][N] for epilogue 0 (identity) and 1 (exact
 *             GELU), fp32 [M][N] for 2 (out += result: residual add) and
 *             5 (fp32 store).
 *  block_n    output tile width: 128, 160, 192, 256, or 320 (CTA pairs only);
 *             N % block_n == 0.
 *  cta_pair   0: one CTA per 128 x block_n tile; 1: CTA pairs (cluster of
 *             2) on 256 x block_n tiles, as the forward uses.
 *  K % 64 == 0; A, B and bias 16-byte aligned (INVALID_ARG otherwise: the
 *  epilogue reads bias four floats at a time).  Enqueued on the handle's
 *  stream. */
moss_enc_status moss_enc_gemm(moss_enc *h, const void *A, const void *B, const float *bias, void *out,
                              int M, int N, int K, int epilogue, int block_n, int cta_pair);

/* The same GEMM with a 4-bit B (the form the linear layers take with
 * cfg.weight_bits = 4): B is given as
 *  Bq         device uint8 [N][K/2]: codes q + 8 of B[n][k], two per byte, the
 *             even k in the low nibble;
 *  Bs         device fp32 [K/128][N]: the scale of each group of 128 k;
 * and the product uses B[n][k] = bf16(fp32(q * s)).  block_n 128, 160, 256
 * or 320, CTA pairs only; K % 128 == 0; epilogues as moss_enc_gemm; A, Bq,
 * Bs and bias 16-byte aligned. */
moss_enc_status moss_enc_gemm_q4(moss_enc *h, const void *A, const void *Bq, const float *Bs, const float *bias,
                                 void *out, int M, int N, int K, int epilogue, int block_n);

/* The same GEMM on e4m3 operands (the form the q/k/v and fc1 GEMMs take with
 * cfg.fp8 = 1): A8 device uint8 [M][K] and B8 device uint8 [N][K] (e4m3
 * bits), sa device fp32 [M], sb device fp32 [N];
 *   out[m][n] = epi((sum_k A8 B8) * sa[m] * sb[n] + bias[n]),
 * epilogue 0 (bf16 out) or 1 (GELU, bf16 out); block_n 128 or 256 (CTA
 * pairs); K % 256 == 0; A8, B8, sb and bias 16-byte aligned. */
moss_enc_status moss_enc_gemm_f8(moss_enc *h, const void *A8, const void *B8, const float *sa, const float *sb,
                                 const float *bias, void *out, int M, int N, int K, int epilogue, int block_n);

/* The same GEMM on NVFP4 operands (page "Ossicle-4B", section "Quantized:
 * NVFP4 and INT4 in vLLM"):
 *  A4, B4     device uint8 [M][K/2], [N][K/2]: E2M1 codes (sign bit 3,
 *             magnitude index 0..7 of 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per
 *             byte, the even k in the low nibble;
 *  sfa, sfb   device uint8: the E4M3 scale of every 16 k of every row, in
 *             512-byte atoms of 128 rows x 64 k ordered [rows/128][K/64]
 *             (rows padded to a multiple of 128), row r of an atom at byte
 *             (r % 32) * 16 + (r / 32) * 4 + (k % 64) / 16;
 *  ga [M], gb [N] device fp32 factors (a row's and the weight's g);
 *   out[m][n] = epi((sum_k a[m][k] b[n][k]) * ga[m] * gb[n] + bias[n]),
 * a and b the E2M1 values times their block scales.  epilogue 0 (bf16 out)
 * or 1 (GELU, bf16 out); 128 x 128 tiles on one CTA each; K % 256 == 0,
 * N % 128 == 0; A4, B4, sfa, sfb, gb and bias 16-byte aligned. */
moss_enc_status moss_enc_gemm_nvf4(moss_enc *h, const void *A4, const void *sfa, const float *ga, const void *B4,
                                   const void *sfb, const float *gb, const float *bias, void *out, int M, int N,
                                   int K, int epilogue);

/* The NVFP4 quantisation of activation rows of 1280 (what the LayerNorm
 * kernel of an NVFP4 handle applies after the norm), on rows given as they
 * are: x device fp32 [M][1280]; codes device uint8 [M][640], sfa device
 * uint8 [ceil(M/128)][20][512] (layout of moss_enc_gemm_nvf4; the bytes of
 * rows >= M in the last block are left as they are), g device fp32 [M].
 * Enqueued on the handle's stream. */
moss_enc_status moss_enc_nvf4_quant_rows(moss_enc *h, const float *x, void *codes, void *sfa, float *g, int M);

/* The NVFP4 quantisation moss_enc_create applies to the q/k/v and fc1
 * weights of an NVFP4 handle, on the host (no device, no handle): w host
 * bf16 bits [n][k], in `parts` equal row ranges with one g each (3 for the
 * fused q/k/v matrix, 1 for fc1); codes host uint8 [n][k/2], sfa host uint8
 * [n/128][k/64][512] (the layout of moss_enc_gemm_nvf4), g host fp32 [n]
 * (each row's part's g).  n/parts % 128 == 0, k % 64 == 0; INVALID_ARG
 * otherwise. */
moss_enc_status moss_enc_nvf4_quant_weights(const void *w, int n, int k, int parts, void *codes, void *sfa, float *g);

/* The GEMM epilogues and conv1 evaluate GELU's erf with a short rational
 * approximation (Abramowitz & Stegun 7.1.28, error <= 3e-7), one value at a
 * time and in pairs (paired fp32 instructions).  This runs both forms
 * against CUDA's erff on 4M points in [-12, 12] and returns the largest
 * |difference| / max(1, |x|) of the GELU values.  Synchronises. */
moss_enc_status moss_enc_selftest_gelu(moss_enc *h, float *max_rel_err);

/* Failure-path check: enqueues a kernel whose one bounded wait can never be
 * satisfied, with a limit of limit_ms (1..2000).  The next
 * moss_enc_synchronize returns MOSS_ENC_ERR_DEVICE_TIMEOUT and clears the
 * flag; the context stays usable. */
moss_enc_status moss_enc_selftest_timeout(moss_enc *h, int limit_ms);

/* ------------------------------------------------- allocation-free log-mel */

/* The source pages describe no such call; it exists for callers that cannot
 * allocate device memory.  Examples: a process whose GPU memory is owned by
 * another framework's pool (a raw cudaMalloc there can fail under pressure or
 * force the pool to release its cache), or a real-time audio front end that
 * must not allocate once it is running.  moss_enc_create allocates the
 * weights and a workspace, so such callers use this call instead: it needs
 * no handle and never allocates.
 *
 * It computes the same Whisper log-mel as moss_enc_logmel for up to
 * MOSS_ENC_STATIC_MAX_CLIPS clips.  Its scratch (the filterbank and FFT
 * tables, per-clip range descriptors and per-clip maxima; 24 KiB) is one
 * statically sized device array inside the library, which every GPU that
 * loads the library keeps until the process exits.
 *  clips        host [n_clips]; same fields and range rules as moss_enc_clip.
 *  mel_out      host array of n_clips device pointers, each fp32
 *               [frames of that clip's range][128] (may be NULL for an empty
 *               range).
 *  log_max_out  device float [n_clips] receiving each clip's log-mel maximum,
 *               or NULL.
 *  stream       cudaStream_t to enqueue on.
 * Returns MOSS_ENC_ERR_CAPACITY when n_clips exceeds MOSS_ENC_STATIC_MAX_CLIPS
 * and MOSS_ENC_ERR_INVALID_ARG for a bad pointer or range (a clip with
 * n_samples > 0 needs its pcm even when its range is empty, because the
 * whole-clip maximum reads it) or when the stream is being captured.
 * The first call on a device sets the scratch up (finds the array's device
 * address and fills the tables, synchronously).  No call may be made while
 * its stream is being captured into a CUDA graph: each call copies its
 * per-clip descriptors from host memory that lives only for the call, so the
 * call refuses a capturing stream (INVALID_ARG) and enqueues nothing.  All calls share the one array, and each call
 * overwrites what the previous call left there: calls whose work overlaps on
 * the GPU (different streams, or several host threads) race and must be
 * serialised by the caller. */
#define MOSS_ENC_STATIC_MAX_CLIPS 64
moss_enc_status moss_enc_logmel_static(const moss_enc_clip *clips, int n_clips, float *const *mel_out,
                                       float *log_max_out, void *stream);

/* ------------------------------------------------------------ measurement */

/* Per-kernel timing by kernel category, taken with CUDA events recorded on the
 * handle's stream around every launch while profiling is enabled. */
typedef struct {
    char name[32];     /* kernel category, e.g. "gemm_fc1" */
    int64_t launches;  /* launches since the last read */
    double ms;         /* summed device time of those launches */
    double flops;      /* summed algorithmic flops (padding not counted) */
    double bytes;      /* summed algorithmic HBM bytes (compulsory reads + writes) */
} moss_enc_kernel_stat;

/* max_launches > 0 enables profiling with room for that many launches
 * between reads (host-side events are created here); 0 disables it. */
moss_enc_status moss_enc_profile_enable(moss_enc *h, int max_launches);

/* Synchronises, aggregates the recorded launches by category into out
 * (up to max entries), clears the record, and returns the number of
 * categories written (negative on error). */
int moss_enc_profile_read(moss_enc *h, moss_enc_kernel_stat *out, int max);

/* Kernels this handle has launched since create (all calls). */
int64_t moss_enc_launch_count(const moss_enc *h);

#ifdef __cplusplus
}
#endif

#endif /* MOSS_ENC_H */
