// Reversal of the token order of [batch*heads][seq][dim] tensors.
//
// The dK and dV passes of the prefill gradient run the block recurrence
// backward in time; the tensor-core prefill kernel only walks forward, so
// those passes read token-reversed copies of their operands and their outputs
// are put back in order afterwards. Both kernels move 16-byte words, coalesced
// along a row, with grid-stride loops sized to the SM count; they are bound by
// HBM bandwidth (one read and one write per word).
#pragma once

#include "common.cuh"

namespace la {

constexpr int kRevThreads = 256;
constexpr int kRevBlocksPerSm = 8;

// dst row (bh, seq-1-i) = src row (bh, i); a row is row_words 16-byte words.
__global__ void __launch_bounds__(kRevThreads)
reverse_rows_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, long long rows, int seq, int row_words) {
    const long long n = rows * row_words;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
        const long long row = e / row_words;
        const int w = (int)(e - row * row_words);
        const long long bh = row / seq;
        const int i = (int)(row - bh * seq);
        dst[(bh * seq + (seq - 1 - i)) * row_words + w] = __ldcs(src + e);
    }
}

// In place: rows i and seq-1-i of every (bh) swap, for i < seq/2.
__global__ void __launch_bounds__(kRevThreads)
reverse_rows_inplace_kernel(uint4 *buf, long long bh_count, int seq, int row_words) {
    const int half = seq / 2;
    const long long per_bh = (long long)half * row_words;
    const long long n = bh_count * per_bh;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
        const long long bh = e / per_bh;
        const long long rem = e - bh * per_bh;
        const int i = (int)(rem / row_words);
        const int w = (int)(rem - (long long)i * row_words);
        uint4 *a = buf + (bh * seq + i) * row_words + w;
        uint4 *b = buf + (bh * seq + (seq - 1 - i)) * row_words + w;
        const uint4 x = *a, y = *b;
        *a = y;
        *b = x;
    }
}

}  // namespace la
