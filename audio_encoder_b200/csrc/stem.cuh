// Conv2D stem helpers (page "MOSS-Transcribe-preview-2B - GGUF",
// "Architecture" table, Conv front-end row): conv1 (1 -> 480 channels, 3x3,
// stride 2, padding 1, GELU) on CUDA cores, and the gather that lays out the
// 3x3 x 480-channel patches of conv2/conv3 as GEMM rows for the tensor cores.
//
// Activations are NHWC per 800-frame chunk: [chunk][time][freq][480] bf16.
#pragma once

#include "common.cuh"

namespace moss {

struct StemChunk {
    int clip;       // clip slot (for the log-mel maximum)
    int mel_row;    // first row of this chunk in the raw log-mel buffer
    int nframes;    // valid frames (1..800); the rest of the chunk is zero
    int pad;
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
    const int t = blockIdx.x, ci = blockIdx.y;
    const StemChunk ch = chunks[ci];
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
    const int c = 2 * threadIdx.x;
    float wa[9], wb[9];
#pragma unroll
    for (int k = 0; k < 9; k++) {
        wa[k] = w1[c * 9 + k];
        wb[k] = w1[(c + 1) * 9 + k];
    }
    const float ba = b1[c], bb = b1[c + 1];
    bf16 *dst = out + ((size_t)ci * 400 + t) * 64 * 480 + c;
#pragma unroll 4
    for (int f = 0; f < 64; f++) {
        float sa = ba, sb = bb;
#pragma unroll
        for (int kf = 0; kf < 3; kf++)
#pragma unroll
            for (int kt = 0; kt < 3; kt++) {
                const float x = in[kt][2 * f + kf];  // freq index 2f + kf - 1, shifted by the pad
                sa += wa[kf * 3 + kt] * x;
                sb += wb[kf * 3 + kt] * x;
            }
        *reinterpret_cast<uint32_t *>(dst + (size_t)f * 480) = pack_bf16x2(gelu_erf(sa), gelu_erf(sb));
    }
}

// Patch gather for a 3x3 stride-2 padding-1 conv over NHWC input
// [chunks][Ti][Fi][480]: row (chunk, to, fo) of the output matrix holds, for
// tap = kf*3 + kt, the 480 input channels of pixel (2to+kt-1, 2fo+kf-1) at
// columns tap*512 .. tap*512+479 (zeros outside the plane and in the 32 pad
// columns).  One thread moves 8 channels (16 bytes).
__global__ void im2col_s2_kernel(const bf16 *__restrict__ in, int Ti, int Fi, long long rows,
                                 bf16 *__restrict__ out)
{
    const int To = (Ti + 1) / 2, Fo = (Fi + 1) / 2;
    const long long total = rows * (9 * 64);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long row = i / (9 * 64);
        const int rem = (int)(i - row * (9 * 64));
        const int tap = rem / 64, c8 = rem % 64;
        const int kf = tap / 3, kt = tap % 3;
        const long long chunk = row / ((long long)To * Fo);
        const int pix = (int)(row - chunk * To * Fo);
        const int to = pix / Fo, fo = pix % Fo;
        const int ti = 2 * to + kt - 1, fi = 2 * fo + kf - 1;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (c8 < 60 && ti >= 0 && ti < Ti && fi >= 0 && fi < Fi)
            v = *reinterpret_cast<const uint4 *>(in + (((size_t)chunk * Ti + ti) * Fi + fi) * 480 + c8 * 8);
        *reinterpret_cast<uint4 *>(out + (size_t)row * 4608 + tap * 512 + c8 * 8) = v;
    }
}

}  // namespace moss
