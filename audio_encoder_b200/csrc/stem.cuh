// Conv2D stem helpers (page "MOSS-Transcribe-preview-2B - GGUF",
// "Architecture" table, Conv front-end row): conv1 (1 -> 480 channels, 3x3,
// stride 2, padding 1, GELU) on CUDA cores.  conv2 and conv3 are implicit
// GEMMs on the tensor cores (gemm.cuh, A_CONV_S2).
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

// conv1 over the normalised log-mel of a chunk.  Input plane (freq 128, time
// 800), with frames >= nframes zero (the tail padding) and conv padding 1.
// Output [chunk][400][64][480] bf16.  One CTA of 240 threads per (pair of
// time steps, chunk): thread j takes time step 2 blockIdx.x + j / 120 and the
// four channels 4 (j % 120) .. +3, two by two in the paired fp32
// instructions.  The five input frames the pair reads sit in shared memory,
// normalised on load, column 2 + f holding frequency f and column 1 the
// conv's zero pad, so that each output frequency step reads its two new
// input columns of a row as one 8-byte word.
__global__ void __launch_bounds__(240) conv1_kernel(const float *__restrict__ mel_raw,
                                                    const StemChunk *__restrict__ chunks,
                                                    const int *__restrict__ gmax_ord,
                                                    const float *__restrict__ w1,  // [480][9] (kf*3+kt)
                                                    const float *__restrict__ b1,  // [480]
                                                    bf16 *__restrict__ out)
{
    __shared__ __align__(16) float in[5][132];  // row r = frame 2 t0 - 1 + r
    grid_dep_wait();
    grid_dep_launch();
    const int t0 = 2 * blockIdx.x, ci = blockIdx.y;
    const StemChunk ch = chunks[ci];
    if (t0 >= ch.t1_lim) return;  // outside the receptive field of the chunk's tokens
    const float floor_v = ordered_to_float(gmax_ord[ch.clip]) - 8.0f;
    for (int i = threadIdx.x; i < 5 * 132; i += blockDim.x) {
        const int r = i / 132, col = i - 132 * r, f = col - 2;
        const int ti = 2 * t0 - 1 + r;
        float v = 0.0f;
        if (f >= 0 && f < 128 && ti >= 0 && ti < ch.nframes) {
            const float x = mel_raw[(size_t)(ch.mel_row + ti) * 128 + f];
            v = (fmaxf(x, floor_v) + 4.0f) * 0.25f;
        }
        in[r][col] = v;
    }
    __syncthreads();
    const int tl = threadIdx.x / 120, t = t0 + tl;
    if (t >= ch.t1_lim) return;  // no barrier follows
    const int c = 4 * (threadIdx.x - 120 * tl);
    float2 wa[9], wb[9];  // channels (c, c+1) and (c+2, c+3)
#pragma unroll
    for (int k = 0; k < 9; k++) {
        wa[k] = make_float2(w1[c * 9 + k], w1[(c + 1) * 9 + k]);
        wb[k] = make_float2(w1[(c + 2) * 9 + k], w1[(c + 3) * 9 + k]);
    }
    const float2 ba = make_float2(b1[c], b1[c + 1]), bb = make_float2(b1[c + 2], b1[c + 3]);
    const float *row[3] = {in[2 * tl], in[2 * tl + 1], in[2 * tl + 2]};  // frames 2t - 1 + kt
    bf16 *dst = out + ((size_t)ci * 400 + t) * 64 * 480 + c;
    // window of output frequency f: columns 2f+1, 2f+2, 2f+3 (frequencies 2f-1 .. 2f+1)
    float x0[3], x1[3], x2[3];
#pragma unroll
    for (int kt = 0; kt < 3; kt++) x2[kt] = row[kt][1];
#pragma unroll 2
    for (int f = 0; f < 64; f++) {
#pragma unroll
        for (int kt = 0; kt < 3; kt++) {
            x0[kt] = x2[kt];
            const float2 n = *reinterpret_cast<const float2 *>(row[kt] + 2 * f + 2);
            x1[kt] = n.x;
            x2[kt] = n.y;
        }
        float2 sa = ba, sb = bb;
#pragma unroll
        for (int kf = 0; kf < 3; kf++)
#pragma unroll
            for (int kt = 0; kt < 3; kt++) {
                const float x = kf == 0 ? x0[kt] : kf == 1 ? x1[kt] : x2[kt];
                sa = __ffma2_rn(wa[kf * 3 + kt], make_float2(x, x), sa);
                sb = __ffma2_rn(wb[kf * 3 + kt], make_float2(x, x), sb);
            }
        const float2 ga = gelu2(sa), gb = gelu2(sb);
        *reinterpret_cast<uint2 *>(dst + (size_t)f * 480) = make_uint2(pack_bf16x2(ga.x, ga.y), pack_bf16x2(gb.x, gb.y));
    }
}

}  // namespace moss
