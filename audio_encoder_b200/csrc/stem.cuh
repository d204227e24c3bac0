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
// Output [chunk][400][64][480] bf16.  One CTA per (time step, chunk); thread
// j owns channels 2j, 2j+1.
__global__ void __launch_bounds__(240) conv1_kernel(const float *__restrict__ mel_raw,
                                                    const StemChunk *__restrict__ chunks,
                                                    const int *__restrict__ gmax_ord,
                                                    const float *__restrict__ w1,  // [480][9] (kf*3+kt)
                                                    const float *__restrict__ b1,  // [480]
                                                    bf16 *__restrict__ out)
{
    __shared__ float in[3][130];  // 3 time rows x (128 freq + 2 zero pads)
    grid_dep_wait();
    grid_dep_launch();
    const int t = blockIdx.x, ci = blockIdx.y;
    const StemChunk ch = chunks[ci];
    if (t >= ch.t1_lim) return;  // outside the receptive field of the chunk's tokens
    const float floor_v = ordered_to_float(gmax_ord[ch.clip]) - 8.0f;
    for (int i = threadIdx.x; i < 3 * 130; i += blockDim.x) {
        const int kt = i / 130, f = i % 130 - 1;
        const int ti = 2 * t + kt - 1;
        float v = 0.0f;
        if (f >= 0 && f < 128 && ti >= 0 && ti < ch.nframes) {
            const float x = mel_raw[(size_t)(ch.mel_row + ti) * 128 + f];
            v = (fmaxf(x, floor_v) + 4.0f) * 0.25f;
        }
        in[kt][i % 130] = v;
    }
    __syncthreads();
    // channels c, c + 1 side by side in the paired fp32 instructions
    const int c = 2 * threadIdx.x;
    float2 w[9];
#pragma unroll
    for (int k = 0; k < 9; k++) w[k] = make_float2(w1[c * 9 + k], w1[(c + 1) * 9 + k]);
    const float2 b = make_float2(b1[c], b1[c + 1]);
    bf16 *dst = out + ((size_t)ci * 400 + t) * 64 * 480 + c;
#pragma unroll 4
    for (int f = 0; f < 64; f++) {
        float2 acc = b;
#pragma unroll
        for (int kf = 0; kf < 3; kf++)
#pragma unroll
            for (int kt = 0; kt < 3; kt++) {
                const float x = in[kt][2 * f + kf];  // freq index 2f + kf - 1, shifted by the pad
                acc = __ffma2_rn(w[kf * 3 + kt], make_float2(x, x), acc);
            }
        const float2 g = gelu2(acc);
        *reinterpret_cast<uint32_t *>(dst + (size_t)f * 480) = pack_bf16x2(g.x, g.y);
    }
}

}  // namespace moss
