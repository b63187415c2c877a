// Single-token Lightning Attention decode step: a bandwidth-bound stream over
// the fp32 per-head states.
//
// For each (batch, head) with slope s ("MINIMAX SIGNAL LAB · M1", §03: the
// recursive fixed-size KV state; §04: FP32 state per head):
//     S <- e^{-s} S + k^T v        (in place)
//     o  = q S
// Each CTA owns one (batch, head) state of D x D floats. Thread (rg, cg) owns
// rows rg*RPT .. rg*RPT+RPT-1 and columns 4cg .. 4cg+3; a warp therefore walks
// whole contiguous rows with 16-byte loads. All RPT loads of a thread are
// issued before any use so that every CTA keeps D*D*4 bytes in flight. The
// column sums of q_r S[r][:] are reduced across row groups in shared memory.
// States are touched exactly once per step, so loads and stores use the
// streaming (evict-first) cache hints.
#pragma once

#include "common.cuh"

namespace la {

constexpr int kDecodeThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const float *__restrict__ slopes, int heads, float *__restrict__ state,
              T *__restrict__ o) {
    constexpr int CG = D / 4;                 // column groups of four
    constexpr int RG = kDecodeThreads / CG;   // row groups
    constexpr int RPT = D / RG;               // rows per thread
    __shared__ float part[RG][D];

    const size_t bh = blockIdx.x;
    const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
    const float decay = decay_pow(slopes[bh % heads], 1.f);
    float4 *S = reinterpret_cast<float4 *>(state + bh * D * D);
    const T *qh = q + bh * D, *kh = k + bh * D, *vh = v + bh * D;

    float4 st[RPT];
#pragma unroll
    for (int u = 0; u < RPT; ++u) st[u] = __ldcs(&S[(size_t)(rg * RPT + u) * CG + cg]);

    const float v0 = to_f32(vh[4 * cg + 0]), v1 = to_f32(vh[4 * cg + 1]);
    const float v2 = to_f32(vh[4 * cg + 2]), v3 = to_f32(vh[4 * cg + 3]);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
        const int row = rg * RPT + u;
        const float kr = to_f32(kh[row]), qr = to_f32(qh[row]);
        float4 x = st[u];
        x.x = fmaf(decay, x.x, kr * v0);
        x.y = fmaf(decay, x.y, kr * v1);
        x.z = fmaf(decay, x.z, kr * v2);
        x.w = fmaf(decay, x.w, kr * v3);
        __stcs(&S[(size_t)row * CG + cg], x);
        a0 = fmaf(qr, x.x, a0); a1 = fmaf(qr, x.y, a1);
        a2 = fmaf(qr, x.z, a2); a3 = fmaf(qr, x.w, a3);
    }
    part[rg][4 * cg + 0] = a0; part[rg][4 * cg + 1] = a1;
    part[rg][4 * cg + 2] = a2; part[rg][4 * cg + 3] = a3;
    __syncthreads();
    if (threadIdx.x < D) {
        float sum = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) sum += part[g][threadIdx.x];
        o[bh * D + threadIdx.x] = from_f32<T>(sum);
    }
}

}  // namespace la
