// Blockwise Lightning Attention prefill on CUDA cores (fp32 arithmetic).
//
// Follows "MINIMAX SIGNAL LAB · M1", §03 Lightning Attention, block by block:
//   O_t = [(Q_t K_t^T) ⊙ D] V_t + (Q_t ⊙ d_q) S_{t-1}
//   S_t = e^{-s m} S_{t-1} + (K_t ⊙ d_k)^T V_t
// with D_ij = e^{-s(i-j)} 1[i>=j], d_q[i] = e^{-s(i+1)}, d_k[j] = e^{-s(m-1-j)}
// and m the block's length (the last block may be short).
//
// This is the general kernel: float32 or bfloat16 inputs, any block length,
// head dims 64 and 128, all arithmetic in fp32. One CTA owns one (batch, head)
// and a 32-wide slice of value columns, so it keeps S_{t-1}[:, slice] (dim x 32
// fp32) in shared memory across the whole sequence; output columns are
// independent, so the slices never talk to each other.
#pragma once

#include "common.cuh"

namespace la {

constexpr int kSimtThreads = 256;
constexpr int kSimtCols = 32;   // value columns per CTA
constexpr int kSimtRows = 32;   // query / key rows per chunk

template <int D>
constexpr size_t simt_smem_bytes() {
    return sizeof(float) * (D * kSimtCols              // S slice
                            + kSimtRows * (D + 1)      // Q chunk (padded rows)
                            + kSimtRows * (D + 1)      // K chunk (padded rows)
                            + kSimtRows * kSimtCols    // V chunk slice
                            + kSimtRows * (kSimtRows + 1));  // P chunk
}

// How one launch maps its tokens and states. The forward prefill is the
// identity pass. The gradients of a prefill are the same block recurrence on
// permuted operands (lightning_api.cu): the dQ pass runs forward with the
// carried state transposed, the dK and dV passes run backward in time with
// the state gradient seen from the last token on.
struct SimtPass {
    int reverse;         // 1: visit tokens from the last to the first
    int state_in_t;      // 1: state_in holds the transpose of the carried state
    int state_shift;     // 1: the first visited token sees the carried state with e^0, not e^{-s}
    int state_out_step;  // 1: write e^{-s} times the final state
};

// Copy `rows` rows (zero-filled up to kSimtRows) of a [*, D] row-major tensor
// into shared memory with padded row stride D+1; source row r is at
// src + r * stride (stride -D walks backward).
template <typename T, int D>
__device__ __forceinline__ void simt_load_rows(float *dst, const T *src, int rows, long stride = D) {
    for (int e = threadIdx.x; e < kSimtRows * D; e += kSimtThreads) {
        const int r = e / D, c = e % D;
        dst[r * (D + 1) + c] = (r < rows) ? to_f32(src[(long)r * stride + c]) : 0.f;
    }
}

template <typename T, int D, bool kGeneral = false>
__global__ void __launch_bounds__(kSimtThreads)
prefill_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float *__restrict__ slopes, int heads, int seq, int block,
                    const float *state_in, T *__restrict__ o, float *state_out, Snapshots sn,
                    SimtPass pass) {
    extern __shared__ float smem[];
    float *S = smem;                               // [D][32]
    float *Qs = S + D * kSimtCols;                 // [32][D+1]
    float *Ks = Qs + kSimtRows * (D + 1);          // [32][D+1]
    float *Vs = Ks + kSimtRows * (D + 1);          // [32][32]
    float *Ps = Vs + kSimtRows * kSimtCols;        // [32][33]

    constexpr int kSlices = D / kSimtCols;
    const int col0 = (blockIdx.x % kSlices) * kSimtCols;  // first value column of this CTA
    const size_t bh = blockIdx.x / kSlices;
    const float s = slopes[bh % heads];
    const T *qh = q + bh * seq * D;
    const T *kh = k + bh * seq * D;
    const T *vh = v + bh * seq * D;
    T *oh = o + bh * seq * D;

    // token x of the visiting order lives in row prow(x) of the tensors
    const bool rev = kGeneral && pass.reverse;
    auto prow = [&](int x) -> long { return rev ? (long)seq - 1 - x : (long)x; };
    const long rstride = rev ? -(long)D : (long)D;
    const float shift = kGeneral ? (float)pass.state_shift : 0.f;

    const int tid = threadIdx.x;
    // output / P mapping: row r, four adjacent columns starting at c4
    const int r = tid / 8, c4 = (tid % 8) * 4;
    // state mapping: rows x = tid/8 + 32u, columns c4..c4+3
    constexpr int kStateRowsPerThread = D / 32;

    for (int e = tid; e < D * kSimtCols; e += kSimtThreads) {
        const int x = e / kSimtCols, c = e % kSimtCols;
        const size_t at = (kGeneral && pass.state_in_t) ? (size_t)(col0 + c) * D + x : (size_t)x * D + col0 + c;
        S[e] = state_in ? state_in[bh * D * D + at] : 0.f;
    }
    __syncthreads();

    for (int t0 = 0; t0 < seq; t0 += block) {
        const int m = min(block, seq - t0);
        for (int i0 = 0; i0 < m; i0 += kSimtRows) {
            const int rows_q = min(kSimtRows, m - i0);
            simt_load_rows<T, D>(Qs, qh + prow(t0 + i0) * D, rows_q, rstride);
            __syncthreads();

            // inter-block term: (q_i ⊙ d_q) S_{t-1}
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int x = 0; x < D; ++x) {
                const float qv = Qs[r * (D + 1) + x];
                const float4 sv = *reinterpret_cast<const float4 *>(&S[x * kSimtCols + c4]);
                acc[0] += qv * sv.x; acc[1] += qv * sv.y; acc[2] += qv * sv.z; acc[3] += qv * sv.w;
            }
            const float dq = decay_pow(s, (float)(i0 + r + 1) - (t0 == 0 ? shift : 0.f));
            for (int u = 0; u < 4; ++u) acc[u] *= dq;

            // intra-block term over key chunks j0 <= last query row of this chunk
            const int last_i = i0 + rows_q - 1;
            for (int j0 = 0; j0 <= last_i; j0 += kSimtRows) {
                const int rows_k = min(kSimtRows, m - j0);
                __syncthreads();  // previous users of Ks / Vs / Ps are done
                simt_load_rows<T, D>(Ks, kh + prow(t0 + j0) * D, rows_k, rstride);
                for (int e = tid; e < kSimtRows * kSimtCols; e += kSimtThreads) {
                    const int jr = e / kSimtCols, c = e % kSimtCols;
                    Vs[e] = (jr < rows_k) ? to_f32(vh[prow(t0 + j0 + jr) * D + col0 + c]) : 0.f;
                }
                __syncthreads();
                // P[r][j] = (q_i . k_j) e^{-s(i-j)} 1[i>=j], four keys per thread
                for (int u = 0; u < 4; ++u) {
                    const int jj = (tid % 8) + 8 * u;
                    float dot = 0.f;
                    for (int x = 0; x < D; ++x) dot += Qs[r * (D + 1) + x] * Ks[jj * (D + 1) + x];
                    const int i = i0 + r, j = j0 + jj;
                    const float w = (j <= i) ? decay_pow(s, (float)(i - j)) : 0.f;
                    Ps[r * (kSimtRows + 1) + jj] = dot * w;
                }
                __syncthreads();
                for (int jj = 0; jj < kSimtRows; ++jj) {
                    const float p = Ps[r * (kSimtRows + 1) + jj];
                    const float4 vv = *reinterpret_cast<const float4 *>(&Vs[jj * kSimtCols + c4]);
                    acc[0] += p * vv.x; acc[1] += p * vv.y; acc[2] += p * vv.z; acc[3] += p * vv.w;
                }
            }
            if (r < rows_q) {
                T *dst = oh + prow(t0 + i0 + r) * D + col0 + c4;
                for (int u = 0; u < 4; ++u) dst[u] = from_f32<T>(acc[u]);
            }
            __syncthreads();
        }

        // state update: S_t = e^{-s m} S_{t-1} + (K_t ⊙ d_k)^T V_t
        const float dblock = decay_pow(s, (float)m - (t0 == 0 ? shift : 0.f));
        for (int u = 0; u < kStateRowsPerThread; ++u) {
            const int x = tid / 8 + 32 * u;
            for (int c = 0; c < 4; ++c) S[x * kSimtCols + c4 + c] *= dblock;
        }
        for (int j0 = 0; j0 < m; j0 += kSimtRows) {
            const int rows_k = min(kSimtRows, m - j0);
            __syncthreads();
            simt_load_rows<T, D>(Ks, kh + prow(t0 + j0) * D, rows_k, rstride);
            for (int e = tid; e < kSimtRows * kSimtCols; e += kSimtThreads) {
                const int jr = e / kSimtCols, c = e % kSimtCols;
                Vs[e] = (jr < rows_k) ? to_f32(vh[prow(t0 + j0 + jr) * D + col0 + c]) : 0.f;
            }
            __syncthreads();
            for (int jj = 0; jj < rows_k; ++jj) {
                const float dk = decay_pow(s, (float)(m - 1 - (j0 + jj)));
                const float4 vv = *reinterpret_cast<const float4 *>(&Vs[jj * kSimtCols + c4]);
                for (int u = 0; u < kStateRowsPerThread; ++u) {
                    const int x = tid / 8 + 32 * u;
                    const float kx = Ks[jj * (D + 1) + x] * dk;
                    float *sp = &S[x * kSimtCols + c4];
                    sp[0] += kx * vv.x; sp[1] += kx * vv.y; sp[2] += kx * vv.z; sp[3] += kx * vv.w;
                }
            }
        }
        __syncthreads();
        // prefix-cache snapshot of S after the first t0 + m tokens
        if (float *snap = snapshot_at(sn, bh, t0 + m, D)) {
            for (int e = tid; e < D * kSimtCols; e += kSimtThreads) {
                const int x = e / kSimtCols, c = e % kSimtCols;
                snap[(size_t)x * D + col0 + c] = S[e];
            }
        }
    }

    if (state_out) {
        const float fo = (kGeneral && pass.state_out_step) ? decay_pow(s, 1.f) : 1.f;
        for (int e = tid; e < D * kSimtCols; e += kSimtThreads) {
            const int x = e / kSimtCols, c = e % kSimtCols;
            state_out[bh * D * D + (size_t)x * D + col0 + c] = fo * S[e];
        }
    }
}

// seq == 0: the state passes through unchanged (zero decay steps).
__global__ void state_passthrough_kernel(const float *state_in, float *state_out, size_t n) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
         e += (size_t)gridDim.x * blockDim.x)
        state_out[e] = state_in ? state_in[e] : 0.f;
}

}  // namespace la
