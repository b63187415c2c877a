// Range guard of the tensor-core prefill.
//
// The tensor-core kernels round the operands they make (P ⊙ D, Q ⊙ d_q, K ⊙ d_k,
// the carried state S and V) to fp16: 11 significant bits, but a range of
// only 2^-24 .. 65504. bf16 inputs span fp32's range, so a head whose inputs
// are large (q . k above 65504 overflows P) or small (the operands fall into
// fp16's subnormals and lose their precision) would come out wrong. The
// blockwise method is linear in v and in the state, and bilinear in q and k,
// so scaling q, k and v by powers of two 2^a, 2^b, 2^c (and the carried state
// by 2^(b+c)) scales o by 2^(a+b+c) and the state by 2^(b+c) exactly, with no
// rounding: the guard picks such exponents per (batch, head).
//
// Pass 1 (the plain kernel) also measures each (batch, head) while it runs, in
// the warps that convert the operands (one packed max per word already in a
// register): the largest |q|, |k| and |v| element and the largest |state_in|
// element. These bound every fp16 operand: |Q ⊙ d_q| <= max|q|,
// |K ⊙ d_k| <= max|k|, |V| <= max|v|, |P ⊙ D| <= d max|q| max|k| (d = 128), and
// each state element |S| <= max|S_in| + max|k| max|v| W, W = the sum over the
// call's tokens of the decay = min(L, 1 / (1 - e^{-s})). A head whose bounds
// keep every operand below 2^15 and its maxima at or above 2^-9 (so that the
// operands' bulk stays in fp16's normal range) is done. Any other head is
// flagged; a second launch (pass 2) takes the verdict and recomputes exactly the
// flagged heads with power-of-two scales, leaving the others alone. Pass 1 learns
// the verdict itself only when the state is carried in place (state_out ==
// state_in): its two CTAs then exchange their maxima, and it does not write the
// final state of a flagged head, which pass 2 still has to read.
//
// Pass 2 first measures the flagged head's largest row norms of q and k (a
// tighter bound on |P ⊙ D| = |q_i . k_j| <= ||q_i|| ||k_j|| than the elementwise
// one, which matters when a few rows are much larger than the rest) and picks
// the exponents from them.
#pragma once

#include <stdint.h>

namespace la {
namespace rg {

// The maxima one of a head's two CTAs measured, over its share of the head's q, k,
// v and state_in (the two shares together cover them: the CTA pair splits the
// rows, the single-CTA kernel's two CTAs the value columns).
struct RangePart {
    float mq;    // largest |q| element
    float mk;    // largest |k| element
    float mv;    // largest |v| element
    float msin;  // largest |state_in| element (0 without a carried-in state)
};
// One record per (batch, head) in the caller's workspace: pass 1 writes the two
// parts, pass 2 combines them, decides, and writes the verdict.
struct RangeRec {
    RangePart part[2];
    int flag;    // written by pass 2: 1 if the head took the scaled recomputation
    int pad[3];
};
static_assert(sizeof(RangeRec) == 48, "RangeRec is 48 bytes");

__device__ __forceinline__ RangePart combine(const RangePart &a, const RangePart &b) {
    return RangePart{fmaxf(a.mq, b.mq), fmaxf(a.mk, b.mk), fmaxf(a.mv, b.mv), fmaxf(a.msin, b.msin)};
}

constexpr float kHi = 32768.f;            // 2^15: every fp16 operand stays below this (fp16 max 65504)
constexpr float kLoElem = 0.001953125f;   // 2^-9: elementwise maxima below this are scaled up
constexpr float kLoQK = 0.0009765625f;    // 2^-10: lower bound on max|q| max|k|
constexpr float kLoKV = 0.000244140625f;  // 2^-12: lower bound on max|k| max|v|

// |a| and |b| compared per half; the larger magnitude (its sign is the xor of
// the two signs, which the final |.| discards)
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Largest value over the warp (non-negative floats order like their bits; a
// NaN, 0x7fc00000 and above, counts as the largest).
__device__ __forceinline__ float warp_max_nonneg(float x) {
    uint32_t r;
    asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(__float_as_uint(x)));
    return __uint_as_float(r);
}

// Sum over the tokens of one call of the per-token decay: min(L, 1 / (1 - e^{-s})).
__device__ __forceinline__ float decay_window(float s, int seq) {
    const float w = s > 0.f ? 1.f / -expm1f(-s) : (float)seq;
    return fminf(w, (float)seq);
}

__device__ __forceinline__ bool finite(float x) { return x == x && fabsf(x) <= 3.0e38f; }

// Pass 1's verdict: true when the plain kernel's fp16 operands all stay below
// 2^15 and its maxima at or above 2^-9. Non-finite maxima (inputs holding inf
// or NaN) keep pass 1's result: scaling cannot make such a result finite.
__device__ __forceinline__ bool plain_ok(const RangePart &r, float s, int seq) {
    if (!finite(r.mq) || !finite(r.mk) || !finite(r.mv) || !finite(r.msin)) return true;
    const float W = decay_window(s, seq);
    const bool hi = fmaxf(fmaxf(r.mq, r.mk), r.mv) <= kHi * 0.5f && 128.f * r.mq * r.mk <= kHi &&
                    r.msin + r.mk * r.mv * W <= kHi;
    const bool lo = fminf(fminf(r.mq, r.mk), r.mv) >= kLoElem && r.mq * r.mk >= kLoQK && r.mk * r.mv >= kLoKV;
    return hi && lo;
}

// floor(log2 x) for a positive finite x (0 otherwise)
__device__ __forceinline__ int ex2floor(float x) {
    if (!(x > 0.f) || !(x <= 3.0e38f)) return 0;
    int e;
    frexpf(x, &e);
    return e - 1;
}

// Pass 2's exponents for q, k and v from the largest row norms nq, nk of q and
// k, the largest |v| and |state_in|: the row norms become [16, 32), the largest
// |v| [4, 8), so |P ⊙ D| <= 2^10 and the bulk of every operand sits well inside
// fp16's normal range. If the state bound (max|S_in| 2^(b+c) + nk max|v| W) then
// passes 2^14, k comes down (and q goes up as much, keeping P's scale) by up to
// 6, then v by the rest. Each exponent stays within [-40, 40], so that every
// factor and o's 2^-(a+b+c) are normal floats; inputs that would need more lie
// outside what the guard serves.
struct Exps {
    int a, b, c;
};
__device__ __forceinline__ Exps scale_exponents(float nq, float nk, float mv, float msin, float s, int seq) {
    Exps e;
    e.a = nq > 0.f ? 4 - ex2floor(nq) : 0;
    e.b = nk > 0.f ? 4 - ex2floor(nk) : 0;
    e.c = mv > 0.f ? 2 - ex2floor(mv) : 0;
    const float W = decay_window(s, seq);
    const float bound = ldexpf(msin, e.b + e.c) + ldexpf(nk, e.b) * ldexpf(mv, e.c) * W;
    if (bound > 16384.f) {
        int excess = ex2floor(bound * (1.f / 16384.f)) + 1;
        const int dk = excess < 6 ? excess : 6;
        e.b -= dk;
        e.a += dk;
        excess -= dk;
        e.c -= excess;
    }
    e.a = max(-40, min(40, e.a));
    e.b = max(-40, min(40, e.b));
    e.c = max(-40, min(40, e.c));
    return e;
}

__device__ __forceinline__ float pow2(int e) { return __int_as_float((127 + e) << 23); }

// Largest sum of squares over rows r0, r0 + step, .. (< seq) of one head's
// [seq][128] bf16 rows in global memory, for the whole CTA: 16 threads per row
// (16 bytes each, fp32 sums), the result reduced over the CTA through `red`
// (one float per warp) and returned to every thread. All threads must call it.
__device__ __forceinline__ float head_max_row_sumsq(const __nv_bfloat16 *rows, int seq, int r0, int step, float *red) {
    const int t = threadIdx.x, warp = t >> 5, half = (t >> 4) & 1, sub = t & 15;
    const int per = blockDim.x >> 4;  // rows per sweep of the CTA
    float best = 0.f;
    // the loop runs alike for both half-warps (their rows differ by `step`), so
    // that every lane takes part in each shuffle
    for (int rw = r0 + step * (2 * warp); rw < seq; rw += step * per) {
        const int r = rw + step * half;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (r < seq) x = __ldg(reinterpret_cast<const uint4 *>(rows + (size_t)r * 128) + sub);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fmaf(bf_lo(w[i]), bf_lo(w[i]), acc);
            acc = fmaf(bf_hi(w[i]), bf_hi(w[i]), acc);
        }
#pragma unroll
        for (int m = 8; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
        best = fmaxf(best, acc);
    }
    const float wmax = warp_max_nonneg(best);
    if ((t & 31) == 0) red[warp] = wmax;
    __syncthreads();
    float m = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
    __syncthreads();
    return m;
}

}  // namespace rg
}  // namespace la
