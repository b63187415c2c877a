// Blockwise Lightning Attention prefill on a CTA pair (cta_group::2): block 256,
// bf16 inputs, head dim 128.
//
// The method ("MINIMAX SIGNAL LAB · M1", §03 Lightning Attention), per block t
// of 256 tokens of one (batch, head) with slope s:
//   O_t = [(Q_t K_t^T) ⊙ D] V_t + (Q_t ⊙ d_q) S_{t-1}
//   S_t = e^{-s m} S_{t-1} + (K_t ⊙ d_k)^T V_t
// D_ij = e^{-s(i-j)} 1[i>=j], d_q[i] = e^{-s(i+1)}, d_k[j] = e^{-s(m-1-j)}.
//
// One cluster of two CTAs works on one (batch, head). The even CTA issues
// every MMA for both SMs with M = 256: A operands are split by rows across
// the pair and B operands by columns, so no product is computed twice.
// CTA c owns
//   - rows 128c .. 128c+127 of every block (its Q sub-tile) and the keys
//     128c .. 128c+127 (its K sub-tile: its half of the B operand of Q K^T),
//   - value columns 64c .. 64c+63 (its half of V, of the state and of the
//     state operand), and
//   - the key-dimension half 64c .. 64c+63 of K ⊙ d_k for the state MMA.
// Per block:
//   QK   SS, M256 N256 K128, bf16       P (128 rows x 256 keys per SM, fp32 in TMEM)
//   QS   TS, M256 N128 K128, f16       O  = Qd S_{t-1}   (Qd = Q ⊙ d_q, fp16 in TMEM)
//   dS   SS, M128 N128 K256, f16       S^T += V^T (K ⊙ d_k) onto e^{-s m} S^T (each
//                                      SM: its 64 value columns x all 128 key dims)
//   PV   TS, M256 N128 K128, f16, twice: O += P V per key half (P ⊙ D, fp16)
// Q K^T runs as one group of 8 MMAs over all 256 keys; its two key halves of P
// are then converted by two warpgroups side by side, and P V takes each half as
// soon as it is converted. (Q K^T as two N = 128 groups, one per half, re-read Q
// from shared memory and took twice the MMA instructions, for no gain.)
// Precision as in the single-CTA kernel: Q K^T on the bf16 inputs; P ⊙ D,
// Q ⊙ d_q, S and K ⊙ d_k rounded to fp16; V widened to fp16 exactly; fp32
// accumulation; the fp32 state stays in TMEM for the whole sequence.
//
// Warp roles (per CTA): warp 0 TMA, warp 1 MMA (even CTA only; the whole warp follows
// the waits and one elected lane issues), warp 2 TMEM,
// warp 3 forwards "Q/K landed" to the even CTA; warpgroup A (warps 4-7) writes
// K ⊙ d_k and widens V, then turns keys 0..127 of P into fp16 P ⊙ D;
// warpgroup B (warps 8-11) builds Qd, then does keys 128..255 of P;
// warpgroup 3 (warps 12-15) carries the state (fp32, in TMEM) and writes O. Hand-offs to the even CTA's MMA thread are
// remote mbarrier arrivals; MMA completions reach both CTAs through
// multicast commits. Every wait is bounded. A barrier that counts arrivals
// from several groups is safe only if no group can arrive for block t+1
// before the barrier's phase for block t has completed; each group's
// per-block sequence below is ordered so that this holds.
//
// Shared memory per CTA (1024-aligned, 128B-swizzled):
//   Q sub-tile 32 KB, K sub-tile 32 KB (keys 128c .. 128c+127),
//   2 stages x (V half for 256 keys 32 KB + K half-dims for 256 keys 32 KB),
//   fp16 state operand 16 KB (rows = this CTA's 64 value columns),
//   output staging 16 KB (half a row block of O, written out by TMA).
// TMEM per CTA: [0,256) P fp32 -> fp16 keys 0..127 in [0,64), keys 128..255
// in [128,192); [256,384) O; [384,448) the fp32 state S^T; [448,512) Qd.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <string>

#include "../../include/lightning.h"
#include "common.cuh"
#include "prefill_tc.cuh"
#include "range_guard.cuh"
#include "tc_ptx.cuh"

namespace la {
namespace pair {

constexpr int kThreads = 512;
constexpr int kDim = 128;
constexpr int kRows = 128;     // rows per CTA per block
constexpr int kBlock = 256;    // tokens per block
constexpr uint32_t kBoxBytes = 16384;   // 128 rows x 64 16-bit values (128 B rows)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + 2 * kBoxBytes;
constexpr uint32_t kOffStage = kOffK + 2 * kBoxBytes;          // 2 stages
constexpr uint32_t kStageBytes = 4 * kBoxBytes;                // V (2 boxes) + Kd (2 boxes)
constexpr uint32_t kOffS = kOffStage + 2 * kStageBytes;
constexpr uint32_t kSBytes = 2 * 8192;                         // 2 boxes of 64 rows x 128 B
constexpr uint32_t kOffE = kOffS + kSBytes;                    // output staging: 128 rows x 64 bf16
constexpr uint32_t kOffBar = kOffE + kBoxBytes;
constexpr int kNumBars = 26;
constexpr uint32_t kOffMisc = (kOffBar + kNumBars * 8 + 15) & ~15u;
constexpr uint32_t kOffGamma = kOffMisc + 64;                  // fused norm + gate: gamma of the head
constexpr uint32_t kSmemBytes = kOffGamma + kDim * 4 + 1024;
static_assert(kOffMisc % 16 == 0 && kOffGamma % 16 == 0, "gamma is read with 16-byte loads");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColP = 0, kColPHi = 128, kColO = 256, kColDS = 384, kColQd = 448;

// barriers: local ones first, then the ones only the even CTA's MMA thread waits on
// (P_CONV, P_FREE: one per key half, index + half)
constexpr int QK_LOADED = 0, VK_LOADED = 1 /* 2 */, P_FULL = 3, QK_DONE = 4, O_FULL = 5,
              DS_FULL = 6, VK_EMPTY = 7 /* 2 */, P_FREE = 9 /* 2 */, QD_LOCAL = 11, QK_FULL = 12,
              QD_READY = 13, S_READY = 14, O_FREE = 15, VK_READY = 16, DS_FREE = 17, P_CONV = 18 /* 2 */,
              DRAIN = 20, G_FULL = 21 /* fused norm + gate: a gate half landed in the staging tile */,
              // range guard (pass 1 only): SCAN_FIN: warpgroups A and B put their maxima of
              // k, v and q in shared memory; SIN_DONE: warpgroup 3 put its maximum of state_in;
              // PEER: the other CTA's maxima landed here; RANGE_DONE: the head's verdict is set
              SCAN_FIN = 22, SIN_DONE = 23, PEER = 24, RANGE_DONE = 25;

// shared-memory words after the barriers
// (the maxima as float bits, which order like unsigned integers for values >= 0)
constexpr uint32_t kMiscTmem = 0, kMiscAbort = 4, kMiscMq = 8, kMiscMk = 12, kMiscMv = 16, kMiscSin = 20,
                   kMiscPeer = 24 /* 4 floats */, kMiscFlag = 40;

constexpr int kBarA = 1, kBarB = 3, kBarW3 = 2;  // named barriers of the three warpgroups

__host__ __device__ constexpr uint32_t idesc(int M, int N, uint32_t fmt, bool a_mn, bool b_mn) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescQK = idesc(256, 256, 1, false, false);  // Q (K-major) x K (K-major), bf16
constexpr uint32_t kIdescQS = idesc(256, 128, 0, false, false);  // Qd (TMEM) x S (K-major), f16
constexpr uint32_t kIdescPV = idesc(256, 128, 0, false, true);   // P (TMEM) x V (MN-major), f16
constexpr uint32_t kIdescDS = idesc(128, 128, 0, true, true);    // V^T (MN-major) x Kd (MN-major), f16

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

using ptx::cluster_rank;
using ptx::cluster_sync;
using ptx::map_to_rank;
// Arrive on the even CTA's copy of barrier `bar`. Every hand-off to the MMA
// thread concerns data in the arriving CTA's own shared memory or TMEM, made
// visible to the tensor core by the async-proxy or tcgen05 fence that precedes
// the arrival, so the default CTA-scope release suffices. A cluster-scope
// release would also drain this thread's outstanding global traffic (the
// output stores), which costs thousands of cycles per hand-off.
__device__ __forceinline__ void arrive_leader(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(map_to_rank(bar, 0)) : "memory");
}

// one lane of a converged warp (the lowest active one)
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(pred));
    return pred != 0;
}

struct Ctx {
    uint8_t *smem;
    uint32_t sbase;
    uint64_t *bars;
    volatile int *abort;
    uint32_t tmem;
};

__device__ __forceinline__ bool wait_bar(const Ctx &c, int idx, uint32_t parity) {
    return ptx::mbar_wait(&c.bars[idx], parity, c.abort);
}
// waits of the even CTA's MMA thread on barriers both CTAs arrive on
__device__ __forceinline__ bool wait_pair(const Ctx &c, int idx, uint32_t parity) {
    return ptx::mbar_wait(&c.bars[idx], parity, c.abort);
}
__device__ __forceinline__ bool group_wait(const Ctx &c, int idx, uint32_t parity, bool leader, int bar_id) {
    const bool ok = leader ? wait_bar(c, idx, parity) : true;
    return ptx::named_bar_and(bar_id, 128, ok);
}
using ptx::mul2;

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float scale) {
    const float2 r = mul2(make_float2(ptx::bf16_lo(w), ptx::bf16_hi(w)), make_float2(scale, scale));
    return ptx::pack_f16(r.x, r.y);
}

// fp32 P columns [col0, col0 + 128) of this thread's row -> fp16 P ⊙ D in
// [dst0, dst0 + 64). Row i (block position) against keys j0 .. j0+127.
// Causal: key j counts for j <= i with e^{-s(i-j)}; anti-causal (upper): for
// j >= i with e^{-s(j-i)}. tab[u] = pscale e^{-s(15-u)}, step = e^{-s};
// pscale is the range guard's factor for P (1 in the plain kernel).
__device__ __forceinline__ void convert_p(uint32_t taddr_row, uint32_t col0, uint32_t dst0, int i, int j0,
                                          float sl2, float step, const float (&tab)[16], bool upper,
                                          float pscale) {
    // 32 fp32 columns per iteration -> 16 fp16 pair columns; the destination
    // [dst0 + 16 q, dst0 + 16 q + 16) lies inside columns already read
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t v[32];
        ptx::tmem_ld32(taddr_row + col0 + 32 * q, v);
        ptx::tmem_ld_wait();
        uint32_t out[16];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const int jb = j0 + 32 * q + 16 * g;
            const int dlast = i - (jb + 15);
            float p[16];
            if (upper) {
                if (jb >= i) {
                    const float wb = ptx::ex2(-sl2 * (float)(jb - i));
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const float2 t = mul2(make_float2(__uint_as_float(v[16 * g + u]), __uint_as_float(v[16 * g + u + 1])),
                                              make_float2(tab[15 - u], tab[14 - u]));
                        const float2 r2 = mul2(t, make_float2(wb, wb));
                        p[u] = r2.x;
                        p[u + 1] = r2.y;
                    }
                } else if (jb + 15 < i) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) p[u] = 0.f;
                } else {
                    // keys from the diagonal (u = i - jb) upward
                    const int d0 = i - jb;
                    float w = pscale;
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const bool live = u >= d0;
                        p[u] = live ? __uint_as_float(v[16 * g + u]) * w : 0.f;
                        w = live ? w * step : w;
                    }
                }
            } else if (dlast >= 0) {
                const float wb = ptx::ex2(-sl2 * (float)dlast);
#pragma unroll
                for (int u = 0; u < 16; u += 2) {
                    const float2 t = mul2(make_float2(__uint_as_float(v[16 * g + u]), __uint_as_float(v[16 * g + u + 1])),
                                          make_float2(tab[u], tab[u + 1]));
                    const float2 r2 = mul2(t, make_float2(wb, wb));
                    p[u] = r2.x;
                    p[u + 1] = r2.y;
                }
            } else if (i < jb) {
#pragma unroll
                for (int u = 0; u < 16; ++u) p[u] = 0.f;
            } else {
                const int d0 = i - jb;
                float w = pscale;
#pragma unroll
                for (int u = 15; u >= 0; --u) {
                    const bool live = u <= d0;
                    p[u] = live ? __uint_as_float(v[16 * g + u]) * w : 0.f;
                    w = live ? w * step : w;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) out[8 * g + u] = ptx::pack_f16(p[2 * u], p[2 * u + 1]);
        }
        __syncwarp();
        ptx::tmem_st16(taddr_row + dst0 + 16 * q, out);
    }
}

// scale one 128-byte swizzled row (64 16-bit values) in place: bf16 -> fp16 x scale.
// kMeasure: also fold the row's largest |value| (bf16, as read) into mx.
template <bool kMeasure>
__device__ __forceinline__ void scale_row_to_f16(uint8_t *row, int r, float scale, uint32_t &mx) {
    uint4 x[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) x[ch] = *reinterpret_cast<const uint4 *>(row + ((ch ^ (r & 7)) << 4));
    if (kMeasure) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
            mx = rg::maxabs_bf16x2(mx, rg::maxabs_bf16x2(rg::maxabs_bf16x2(x[ch].x, x[ch].y),
                                                         rg::maxabs_bf16x2(x[ch].z, x[ch].w)));
    }
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint4 y;
        y.x = bf16x2_to_f16x2(x[ch].x, scale); y.y = bf16x2_to_f16x2(x[ch].y, scale);
        y.z = bf16x2_to_f16x2(x[ch].z, scale); y.w = bf16x2_to_f16x2(x[ch].w, scale);
        *reinterpret_cast<uint4 *>(row + ((ch ^ (r & 7)) << 4)) = y;
    }
}

// Normalisation and gating fused into the output epilogue (per-head RMS
// reading): y[b][l][h*128 + c] = gamma[h*128 + c] o_c / sqrt(mean_c o_c^2 + eps)
// * sigmoid(gate[b][l][h*128 + c]), written token-major in place of o.
struct PairNormGate {
    const __nv_bfloat16 *gate;  // [batch][seq][heads*128]
    const float *gamma;         // [heads*128]
    float eps;
};

// How one launch runs. The forward prefill is {0, 0}; the passes of the
// backward computation (lightning_api.cu) read the carried state transposed,
// or run anti-causal. The direction is a template argument of the kernel, so
// that the causal instantiation carries no anti-causal code (a smaller hot
// loop for the instruction cache).
struct PairPass {
    int state_in_t;  // 1: state_in holds the transpose of the carried state
    int anti;        // 1: anti-causal: blocks from last to first, query i sees keys j >= i
                     //    with e^{-s(j-i)}, the carried state anchored at each block's last
                     //    token (query factor e^{-s(m-1-i)}, key factor e^{-s(j+1)})
};

// kScaled = false: the plain kernel (pass 1 of the range guard), which also
// measures every (batch, head) and records its bounds and verdict in rec[bh].
// kScaled = true: pass 2, which returns at once for a head pass 1 did not flag
// and otherwise recomputes it with the guard's power-of-two operand scales.
template <bool kAnti, bool kNormGate, bool kScaled>
__global__ void __launch_bounds__(kThreads, 1)
prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_g,
                    const float *__restrict__ slopes, int heads, int seq, const float *state_in,
                    float *state_out, Snapshots sn, PairPass pp, PairNormGate ng, rg::RangeRec *rec,
                    const __nv_bfloat16 *qg, const __nv_bfloat16 *kg) {
    extern __shared__ uint8_t smem_raw[];
    // pass 1: pass 2 may be scheduled now (it waits for this grid's completion before
    // reading anything), so that its launch overlaps this one
    if (!kScaled && threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;");
    // operand scales: q, k, v, P = q k, the carried state, its inverse, and o's inverse
    float f_q = 1.f, f_k = 1.f, f_v = 1.f, f_p = 1.f, f_s = 1.f, f_su = 1.f, f_o = 1.f;
    if constexpr (kScaled) {
        // pass 2 is launched as pass 1's programmatic dependent: wait until pass 1 has
        // completed and its records are visible
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int bh0 = blockIdx.x >> 1;
        const rg::RangePart r = rg::combine(rec[bh0].part[0], rec[bh0].part[1]);
        const bool flag = !rg::plain_ok(r, slopes[bh0 % heads], seq);
        if (threadIdx.x == 0 && (blockIdx.x & 1) == 0) rec[bh0].flag = flag ? 1 : 0;
        if (!flag) return;  // both CTAs of the pair read the same record and leave together
        // the head's largest row norms of q and k, fp32 sums: this CTA takes every other
        // row, then the two CTAs exchange through the output staging tile (first written
        // after the set-up's cluster barrier, which the other CTA reaches only after its read)
        const uint32_t a0 = ptx::smem_addr(smem_raw);
        uint8_t *sm = smem_raw + (((a0 + 1023u) & ~1023u) - a0);
        float *red = reinterpret_cast<float *>(sm + kOffE);
        float *mine = reinterpret_cast<float *>(sm + kOffE + 64);
        const uint32_t crank = cluster_rank();
        const size_t hb = (size_t)bh0 * seq * kDim;
        const float sq = rg::head_max_row_sumsq(qg + hb, seq, (int)crank, 2, red);
        const float sk = rg::head_max_row_sumsq(kg + hb, seq, (int)crank, 2, red);
        if (threadIdx.x == 0) {
            mine[0] = sq;
            mine[1] = sk;
        }
        cluster_sync();
        float pq, pk;
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pq) : "r"(map_to_rank(mine, crank ^ 1u)) : "memory");
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pk) : "r"(map_to_rank(mine + 1, crank ^ 1u)) : "memory");
        const float nq = sqrtf(fmaxf(sq, pq)), nk = sqrtf(fmaxf(sk, pk));
        const rg::Exps e = rg::scale_exponents(nq, nk, r.mv, r.msin, slopes[bh0 % heads], seq);
        f_q = rg::pow2(e.a);
        f_k = rg::pow2(e.b);
        f_v = rg::pow2(e.c);
        f_p = rg::pow2(e.a + e.b);
        f_s = rg::pow2(e.b + e.c);
        f_su = rg::pow2(-(e.b + e.c));
        f_o = rg::pow2(-(e.a + e.b + e.c));
    }
    const uint32_t raw_addr = ptx::smem_addr(smem_raw);
    const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
    Ctx c;
    c.smem = smem_raw + pad;
    c.sbase = raw_addr + pad;
    c.bars = reinterpret_cast<uint64_t *>(c.smem + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c.smem + kOffMisc + kMiscTmem);
    c.abort = reinterpret_cast<volatile int *>(c.smem + kOffMisc + kMiscAbort);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int bh = blockIdx.x >> 1;
    const float s = slopes[bh % heads];
    const float sl2 = s * kLog2e;
    const int nblk = (seq + kBlock - 1) / kBlock;
    // block index of the t-th block visited, and its length
    auto tb = [&](int t) { return kAnti ? nblk - 1 - t : t; };
    auto blen = [&](int t) { return min(kBlock, seq - tb(t) * kBlock); };

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) ptx::mbar_init(&c.bars[i], 1);
        // the even CTA's MMA thread collects arrivals from both CTAs
        ptx::mbar_init(&c.bars[QK_FULL], 2);
        ptx::mbar_init(&c.bars[QD_READY], 2);
        ptx::mbar_init(&c.bars[S_READY], 2);
        ptx::mbar_init(&c.bars[O_FREE], 2);
        ptx::mbar_init(&c.bars[VK_READY], 2);
        ptx::mbar_init(&c.bars[DS_FREE], 2);
        ptx::mbar_init(&c.bars[P_CONV], 2);
        ptx::mbar_init(&c.bars[P_CONV + 1], 2);
        ptx::mbar_init(&c.bars[SCAN_FIN], 2);  // warpgroups A and B
        *reinterpret_cast<uint32_t *>(c.smem + kOffMisc + kMiscMq) = 0u;
        *reinterpret_cast<uint32_t *>(c.smem + kOffMisc + kMiscMk) = 0u;
        *reinterpret_cast<uint32_t *>(c.smem + kOffMisc + kMiscMv) = 0u;
        *c.abort = 0;
        *reinterpret_cast<uint32_t *>(c.smem + kOffMisc + kMiscSin) = 0u;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_o);
        if (kNormGate) ptx::prefetch_tensormap(&tm_g);
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    ptx::tc_fence_before();
    __syncthreads();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated on both SMs
    ptx::tc_fence_after();
    c.tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (each CTA)
        if (lane == 0) {
            bool ok = true;
            int vk_issued = 0, qk_issued = 0;
            auto load_vk = [&](int t) -> bool {
                const int st = t & 1;
                if (!wait_bar(c, VK_EMPTY + st, ((uint32_t)(t >> 1) & 1u) ^ 1u)) return false;
                uint8_t *dst = c.smem + kOffStage + st * kStageBytes;
                uint64_t *bar = &c.bars[VK_LOADED + st];
                ptx::mbar_arrive_expect_tx(bar, kStageBytes);
                const int row0 = tb(t) * kBlock;
                ptx::tma_load_3d(dst, &tm_v, bar, 64 * rank, row0, bh);                      // V keys 0..127
                ptx::tma_load_3d(dst + kBoxBytes, &tm_v, bar, 64 * rank, row0 + kRows, bh);  // V keys 128..255
                ptx::tma_load_3d(dst + 2 * kBoxBytes, &tm_k, bar, 64 * rank, row0, bh);      // K dims half, keys 0..127
                ptx::tma_load_3d(dst + 3 * kBoxBytes, &tm_k, bar, 64 * rank, row0 + kRows, bh);
                vk_issued = t + 1;
                return true;
            };
            ok = load_vk(0);
            for (int t = 0; t < nblk && ok; ++t) {
                // Q and K sub-tiles of block t, once block t-1's Q K^T ran and its Qd was built
                if (t > 0) ok = wait_bar(c, QK_DONE, (uint32_t)(t - 1) & 1u) && wait_bar(c, QD_LOCAL, (uint32_t)(t - 1) & 1u);
                if (!ok) break;
                const int row = tb(t) * kBlock + kRows * (int)rank;
                uint64_t *qkbar = &c.bars[QK_LOADED];
                ptx::mbar_arrive_expect_tx(qkbar, 4 * kBoxBytes);
                ptx::tma_load_3d(c.smem + kOffQ, &tm_q, qkbar, 0, row, bh);
                ptx::tma_load_3d(c.smem + kOffQ + kBoxBytes, &tm_q, qkbar, 64, row, bh);
                // K sub-tile: keys 128c .. 128c+127, this CTA's half of the N = 256 B operand
                ptx::tma_load_3d(c.smem + kOffK, &tm_k, qkbar, 0, row, bh);
                ptx::tma_load_3d(c.smem + kOffK + kBoxBytes, &tm_k, qkbar, 64, row, bh);
                qk_issued = t + 1;
                if (t + 1 < nblk) ok = load_vk(t + 1);
            }
            // let every copy issued land before the CTA may exit
            volatile int never = 0;
            if (qk_issued > 0) ptx::mbar_wait(&c.bars[QK_LOADED], (uint32_t)(qk_issued - 1) & 1u, &never);
            for (int t = vk_issued > 2 ? vk_issued - 2 : 0; t < vk_issued; ++t)
                ptx::mbar_wait(&c.bars[VK_LOADED + (t & 1)], (uint32_t)(t >> 1) & 1u, &never);
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ forwarder (each CTA)
        if (lane == 0) {
            for (int t = 0; t < nblk; ++t) {
                if (!wait_bar(c, QK_LOADED, (uint32_t)t & 1u)) break;
                arrive_leader(&c.bars[QK_FULL]);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ range guard (pass 1)
        // With the state carried in place (state_out == state_in), lane 0 combines this
        // CTA's maxima with the other CTA's and sets the verdict here, so that the final
        // state of a head pass 2 will recompute is not overwritten (pass 2 reads it).
        if (!kScaled && lane == 0 && state_out != nullptr && state_out == state_in) {
            const uint32_t *misc = reinterpret_cast<const uint32_t *>(c.smem + kOffMisc);
            float *peer = reinterpret_cast<float *>(c.smem + kOffMisc + kMiscPeer);
            bool ok = wait_bar(c, SCAN_FIN, 0) && wait_bar(c, SIN_DONE, 0);
            if (ok) {
                // this CTA's maxima to the other CTA
                const float v4[4] = {__uint_as_float(misc[kMiscMq / 4]), __uint_as_float(misc[kMiscMk / 4]),
                                     __uint_as_float(misc[kMiscMv / 4]), __uint_as_float(misc[kMiscSin / 4])};
                const uint32_t other = rank ^ 1u;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(map_to_rank(peer + i, other)), "f"(v4[i])
                                 : "memory");
                asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                                 map_to_rank(&c.bars[PEER], other))
                             : "memory");
                ok = ptx::mbar_wait_cluster(&c.bars[PEER], 0, c.abort);
                if (ok) {
                    const rg::RangePart r = rg::combine(rg::RangePart{v4[0], v4[1], v4[2], v4[3]},
                                                        rg::RangePart{peer[0], peer[1], peer[2], peer[3]});
                    *reinterpret_cast<volatile int *>(c.smem + kOffMisc + kMiscFlag) = rg::plain_ok(r, s, seq) ? 0 : 1;
                    ptx::mbar_arrive(&c.bars[RANGE_DONE]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        // the whole warp follows the waits; one elected lane issues the MMAs and commits
        if (rank == 0) {
            const uint32_t tm = c.tmem;
            const uint64_t dq = sdesc(c.sbase + kOffQ, 16u, 1024u);
            const uint64_t dk = sdesc(c.sbase + kOffK, 16u, 1024u);
            const uint64_t ds = sdesc(c.sbase + kOffS, 16u, 1024u);
            const uint64_t dstage = sdesc(c.sbase + kOffStage, kBoxBytes, 1024u);
            bool ok = true;
            for (int t = 0; t < nblk && ok; ++t) {
                const uint32_t par = t & 1, fpar = par ^ 1u;
                const uint64_t vdesc = dstage + (uint64_t)((uint32_t)(t & 1) * (kStageBytes >> 4));
                const uint64_t kddesc = vdesc + (uint64_t)((2 * kBoxBytes) >> 4);
                // P = Q K^T for all 256 keys, once the previous block's P V has read P
                ok = wait_pair(c, QK_FULL, par) && wait_bar(c, P_FREE, fpar) && wait_bar(c, P_FREE + 1, fpar);
                if (!ok) break;
                ptx::tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint64_t koff = (uint64_t)(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4);
                        ptx::mma_ss_2(tm + kColP, dq + koff, dk + koff, kIdescQK, k > 0);
                    }
                    ptx::mma_commit_2_mc(&c.bars[P_FULL], 0x3);
                }
                __syncwarp();
                if (elect_one()) ptx::mma_commit_2_mc(&c.bars[QK_DONE], 0x3);
                __syncwarp();
                // O = Qd S_{t-1}
                ok = wait_pair(c, QD_READY, par) && wait_pair(c, S_READY, par) && wait_pair(c, O_FREE, fpar);
                if (!ok) break;
                ptx::tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint64_t koff = (uint64_t)(((k >> 2) * 8192 + (k & 3) * 32) >> 4);
                        ptx::mma_ts_2(tm + kColO, tm + kColQd + 8u * k, ds + koff, kIdescQS, k > 0);
                    }
                }
                __syncwarp();
                // S^T += V^T (K ⊙ d_k), onto e^{-s m} S^T prepared in TMEM
                ok = wait_pair(c, VK_READY, par) && wait_pair(c, DS_FREE, par);
                if (!ok) break;
                ptx::tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const uint64_t koff = (uint64_t)(k * (2048 >> 4));
                        ptx::mma_ss_2(tm + kColDS, vdesc + koff, kddesc + koff, kIdescDS, 1);
                    }
                    // S_t is complete and S_{t-1} (the operand copy) is no longer read
                    ptx::mma_commit_2_mc(&c.bars[DS_FULL], 0x3);
                }
                __syncwarp();
                // O += P V, one key half at a time
#pragma unroll 1
                for (int h = 0; h < 2 && ok; ++h) {
                    ok = wait_pair(c, P_CONV + h, par);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            ptx::mma_ts_2(tm + kColO, tm + kColPHi * h + 8u * k,
                                          vdesc + (uint64_t)((8 * h + k) * (2048 >> 4)), kIdescPV, 1);
                        ptx::mma_commit_2_mc(&c.bars[P_FREE + h], 0x3);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (elect_one()) {
                    ptx::mma_commit_2_mc(&c.bars[O_FULL], 0x3);
                    ptx::mma_commit_2_mc(&c.bars[VK_EMPTY + (t & 1)], 0x3);
                }
                __syncwarp();
            }
            if (elect_one()) ptx::mma_commit_2_mc(&c.bars[DRAIN], 0x1);
            __syncwarp();
            volatile int never = 0;
            ptx::mbar_wait(&c.bars[DRAIN], 0, &never);
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------------------ warpgroups A and B
        const int grp = (warp - 4) >> 2;           // 0: keys 0..127 (+ K ⊙ d_k), 1: keys 128..255 (+ Qd)
        const int r = (threadIdx.x & 127);         // TMEM lane = row of this CTA's sub-tile
        const bool leader = r == 0;
        const int bar_id = grp == 0 ? kBarA : kBarB;
        const uint32_t trow = c.tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const int i = kRows * (int)rank + r;       // row position inside the block
        const float step = ptx::ex2(-sl2);
        float tab[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) tab[u] = ptx::ex2(-sl2 * (float)(15 - u)) * f_p;
        // pass 1: the largest |x| this thread converts (bf16 pairs; group A: k in mx0 and
        // v in mx1, group B: q in mx0), for the range guard
        uint32_t mx0 = 0u, mx1 = 0u;
        for (int t = 0; t < nblk; ++t) {
            const uint32_t par = t & 1;
            const int m = blen(t);
            if (grp == 0) {
                // K ⊙ d_k (fp16) for this CTA's key-dim half and V widened to fp16, keys r
                // and 128 + r. The
                // wait on the previous block's dS keeps this group from arriving on
                // VK_READY for block t before that barrier's phase t-1 completed
                // (VK_READY counts arrivals from both CTAs' groups).
                if (t > 0 && !group_wait(c, DS_FULL, (uint32_t)(t - 1) & 1u, leader, bar_id)) goto ab_done;
                if (!group_wait(c, VK_LOADED + (t & 1), (uint32_t)(t >> 1) & 1u, leader, bar_id)) goto ab_done;
                uint8_t *vt = c.smem + kOffStage + (t & 1) * kStageBytes;
                uint8_t *kd = vt + 2 * kBoxBytes;
#pragma unroll 1
                for (int u = 0; u < 4; ++u) {
                    // u = 0, 1: K rows r and 128 + r scaled by d_k; u = 2, 3: V rows widened
                    const int h = u & 1, j = kRows * h + r;
                    const float sc = u >= 2   ? f_v
                                     : j >= m ? 0.f
                                              : ptx::ex2(-sl2 * (float)(kAnti ? j + 1 : m - 1 - j)) * f_k;
                    scale_row_to_f16<!kScaled>((u >= 2 ? vt : kd) + h * kBoxBytes + r * 128, r, sc, u >= 2 ? mx1 : mx0);
                }
                ptx::fence_proxy_async_smem();
                ptx::named_bar_sync(bar_id, 128);
                if (leader) arrive_leader(&c.bars[VK_READY]);
            } else {
                // Qd = Q ⊙ d_q (fp16) into TMEM [448, 512), once the previous block's
                // Qd S MMA (which precedes its dS MMA) has read the region
                if (t > 0 && !group_wait(c, DS_FULL, (uint32_t)(t - 1) & 1u, leader, bar_id)) goto ab_done;
                if (!group_wait(c, QK_LOADED, par, leader, bar_id)) goto ab_done;
                const float dq = (kAnti ? (i < m ? ptx::ex2(-sl2 * (float)(m - 1 - i)) : 0.f)
                                          : ptx::ex2(-sl2 * (float)(i + 1))) * f_q;
                const uint8_t *qrow = c.smem + kOffQ + r * 128;
#pragma unroll 1
                for (int hb = 0; hb < 4; ++hb) {
                    uint32_t out[16];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const int chunk = 4 * (hb & 1) + cc;
                        const uint4 q4 = *reinterpret_cast<const uint4 *>(qrow + (hb >> 1) * kBoxBytes +
                                                                          ((chunk ^ (r & 7)) << 4));
                        if (!kScaled)
                            mx0 = rg::maxabs_bf16x2(mx0, rg::maxabs_bf16x2(rg::maxabs_bf16x2(q4.x, q4.y),
                                                                           rg::maxabs_bf16x2(q4.z, q4.w)));
                        out[4 * cc + 0] = bf16x2_to_f16x2(q4.x, dq);
                        out[4 * cc + 1] = bf16x2_to_f16x2(q4.y, dq);
                        out[4 * cc + 2] = bf16x2_to_f16x2(q4.z, dq);
                        out[4 * cc + 3] = bf16x2_to_f16x2(q4.w, dq);
                    }
                    __syncwarp();
                    ptx::tmem_st16(trow + kColQd + 16 * hb, out);
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                ptx::named_bar_sync(bar_id, 128);
                if (leader) {
                    ptx::mbar_arrive(&c.bars[QD_LOCAL]);
                    arrive_leader(&c.bars[QD_READY]);
                }
            }
            // P ⊙ D -> fp16 for keys [128 grp, 128 grp + 128); the quadrant the mask
            // zeroes (causal: rows 0..127 x keys 128..255; anti-causal: rows
            // 128..255 x keys 0..127) is only cleared
            if (!group_wait(c, P_FULL, par, leader, bar_id)) goto ab_done;
            ptx::tc_fence_after();
            if (kAnti ? (grp == 0 && rank == 1) : (grp == 1 && rank == 0)) {
                // every entry of this quadrant is masked
                uint32_t zero[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) zero[u] = 0u;
#pragma unroll
                for (int q = 0; q < 4; ++q) ptx::tmem_st16(trow + (grp == 0 ? kColP : kColPHi) + 16 * q, zero);
            } else {
                convert_p(trow, grp == 0 ? kColP : kColPHi, grp == 0 ? kColP : kColPHi, i, kRows * grp, sl2,
                          step, tab, kAnti, f_p);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            ptx::named_bar_sync(bar_id, 128);
            if (leader) arrive_leader(&c.bars[P_CONV + grp]);
        }
    ab_done:
        if (!kScaled) {
            // the group's maxima into shared memory for the range guard's verdict
            const auto as_float = [](uint32_t w) { return fmaxf(fabsf(rg::bf_lo(w)), fabsf(rg::bf_hi(w))); };
            const float m0 = rg::warp_max_nonneg(as_float(mx0)), m1 = rg::warp_max_nonneg(as_float(mx1));
            if (lane == 0) {
                uint32_t *misc = reinterpret_cast<uint32_t *>(c.smem + kOffMisc);
                atomicMax(misc + (grp == 0 ? kMiscMk : kMiscMq) / 4, __float_as_uint(m0));
                if (grp == 0) atomicMax(misc + kMiscMv / 4, __float_as_uint(m1));
            }
            ptx::named_bar_sync(bar_id, 128);
            if (leader) {
                // this CTA's share of the head's maxima, for pass 2
                const uint32_t *misc = reinterpret_cast<const uint32_t *>(c.smem + kOffMisc);
                rg::RangePart &part = rec[bh].part[rank];
                if (grp == 0) {
                    part.mk = __uint_as_float(misc[kMiscMk / 4]);
                    part.mv = __uint_as_float(misc[kMiscMv / 4]);
                } else {
                    part.mq = __uint_as_float(misc[kMiscMq / 4]);
                }
                ptx::mbar_arrive(&c.bars[SCAN_FIN]);
            }
        }
    } else if (warp >= 12) {
        // ------------------------------------------------------------ warpgroup 3
        // The fp32 state S^T lives in TMEM [384, 448) in the 2x2 layout of the
        // M=128 pair MMA: lane l holds S[64 (l >> 6) + q][64 rank + (l & 63)],
        // q = 0..63. Before each block's state MMA this group leaves e^{-s m} S
        // there, and the MMA adds (K ⊙ d_k)^T V on top.
        const int l = threadIdx.x - 384;
        const bool leader = l == 0;
        const uint32_t trow = c.tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const int vcol = 64 * (int)rank + (l & 63);
        const int khalf = l >> 6;
        const size_t sb = (size_t)bh * kDim * kDim;
        // fp16 state operand: K-major rows = value column (l & 63), 64 key dims per box
        uint8_t *srow = c.smem + kOffS + khalf * 8192 + (l & 63) * 128;
        // fused norm + gate: this head's gamma in shared memory (visible to the group
        // after the first publish's barrier); the gate reaches the output staging tile
        // by TMA, 64 channels x 128 tokens at a time
        const int nb = bh / heads, nh = bh - nb * heads;
        const float *gsm = reinterpret_cast<const float *>(c.smem + kOffGamma);
        if (kNormGate) reinterpret_cast<float *>(c.smem + kOffGamma)[l] = ng.gamma[(size_t)nh * kDim + l];
        // gate half hh of block t into the staging tile, once the previous store has read it
        int g_issued = 0;  // gate loads issued (leader): the k-th completes G_FULL's phase k
        auto load_gate = [&](int t, int hh) {
            ++g_issued;
            ptx::bulk_wait_read();
            ptx::mbar_arrive_expect_tx(&c.bars[G_FULL], kBoxBytes);
            ptx::tma_load_4d(c.smem + kOffE, &tm_g, &c.bars[G_FULL], 64 * hh, nh, tb(t) * kBlock + kRows * (int)rank,
                             nb);
        };
        // one 32-value half of this thread's state row: operand copy, optional
        // prefix-cache snapshot and state_out, then the decayed value back into
        // TMEM for the next MMA
        auto carry_half = [&](const float (&sv)[32], int hh, float dnext, bool last, float *snap, bool write_state) {
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {
                const int ch = 4 * hh + cq;
                uint4 wv;
                wv.x = ptx::pack_f16(sv[8 * cq + 0], sv[8 * cq + 1]);
                wv.y = ptx::pack_f16(sv[8 * cq + 2], sv[8 * cq + 3]);
                wv.z = ptx::pack_f16(sv[8 * cq + 4], sv[8 * cq + 5]);
                wv.w = ptx::pack_f16(sv[8 * cq + 6], sv[8 * cq + 7]);
                *reinterpret_cast<uint4 *>(srow + ((ch ^ (l & 7)) << 4)) = wv;
            }
            if (snap) {
#pragma unroll
                for (int q = 0; q < 32; ++q) snap[(size_t)(64 * khalf + 32 * hh + q) * kDim + vcol] = sv[q] * f_su;
            }
            if (last) {
                if (write_state) {
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        state_out[sb + (size_t)(64 * khalf + 32 * hh + q) * kDim + vcol] = sv[q] * f_su;
                }
            } else {
                uint32_t lo[16], hi[16];
#pragma unroll
                for (int q = 0; q < 16; q += 2) {
                    const float2 a = mul2(make_float2(sv[q], sv[q + 1]), make_float2(dnext, dnext));
                    const float2 bb = mul2(make_float2(sv[16 + q], sv[17 + q]), make_float2(dnext, dnext));
                    lo[q] = __float_as_uint(a.x);
                    lo[q + 1] = __float_as_uint(a.y);
                    hi[q] = __float_as_uint(bb.x);
                    hi[q + 1] = __float_as_uint(bb.y);
                }
                __syncwarp();
                ptx::tmem_st16(trow + kColDS + 32 * hh, lo);
                ptx::tmem_st16(trow + kColDS + 32 * hh + 16, hi);
            }
        };
        auto publish = [&](bool last) {
            if (!last) ptx::tmem_st_wait();
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::named_bar_sync(kBarW3, 128);
            if (leader) {
                arrive_leader(&c.bars[S_READY]);   // operand copy of S ready
                arrive_leader(&c.bars[DS_FREE]);   // e^{-s m} S ready for the next state MMA
            }
        };
        // t = -1 takes the carried-in state; block t >= 0 takes S_t from TMEM
        for (int t = -1; t < nblk; ++t) {
            const uint32_t par = t & 1;
            const bool last = t + 1 == nblk;
            if (kNormGate && t >= 0 && leader) {
                // this block's gate rows into L2 now; the epilogue loads them a block later
                ptx::tma_prefetch_4d(&tm_g, 0, nh, tb(t) * kBlock + kRows * (int)rank, nb);
                ptx::tma_prefetch_4d(&tm_g, 64, nh, tb(t) * kBlock + kRows * (int)rank, nb);
            }
            // S_t is in TMEM once the state MMA is done
            if (t >= 0) {
                if (!group_wait(c, DS_FULL, par, leader, kBarW3)) goto w3_done;
                ptx::tc_fence_after();
            }
            // with the state carried in place (state_out == state_in), pass 1 writes the final
            // state only for a head the range guard passed, so that pass 2 can still read it
            bool write_state = state_out != nullptr;
            if (!kScaled && last && write_state && state_out == state_in) {
                if (!group_wait(c, RANGE_DONE, 0, leader, kBarW3)) goto w3_done;
                write_state = *reinterpret_cast<volatile int *>(c.smem + kOffMisc + kMiscFlag) == 0;
            }
            {
                // decay from block t's end to block t+1's end (from the carried state's
                // position to block 0's end when t = -1)
                const float dnext =
                    last ? 0.f
                         : ptx::ex2(-sl2 * (float)blen(t + 1));
                float *snap = t >= 0 && !kAnti ? snapshot_at(sn, bh, t * kBlock + blen(t), kDim) : nullptr;
                float msin = 0.f;  // pass 1: the largest |state_in| element of this thread
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    float sv[32];
                    if (t >= 0) {
                        uint32_t d[32];
                        ptx::tmem_ld32(trow + kColDS + 32 * hh, d);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 32; ++q) sv[q] = __uint_as_float(d[q]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const float x = state_in ? state_in[sb + (pp.state_in_t
                                                                        ? (size_t)vcol * kDim + (64 * khalf + 32 * hh + q)
                                                                        : (size_t)(64 * khalf + 32 * hh + q) * kDim + vcol)]
                                                     : 0.f;
                            msin = fmaxf(msin, fabsf(x));
                            sv[q] = x * f_s;
                        }
                    }
                    carry_half(sv, hh, dnext, last, snap, write_state);
                }
                publish(last);
                if (!kScaled && t < 0) {
                    // the carried-in state's bound for the range guard
                    const float m = rg::warp_max_nonneg(msin);
                    if ((l & 31) == 0) atomicMax(reinterpret_cast<uint32_t *>(c.smem + kOffMisc + kMiscSin), __float_as_uint(m));
                    ptx::named_bar_sync(kBarW3, 128);
                    if (leader) {
                        rec[bh].part[rank].msin = __uint_as_float(*reinterpret_cast<const uint32_t *>(
                            c.smem + kOffMisc + kMiscSin));
                        ptx::mbar_arrive(&c.bars[SIN_DONE]);
                    }
                }
            }
            if (t < 0) continue;
            if (kNormGate && leader) load_gate(t, 0);
            // O rows of this CTA: TMEM (fp32) -> bf16 -> staging (128B-swizzled) -> TMA
            // store, 64 value columns at a time; rows past seq are clipped by TMA
            if (!group_wait(c, O_FULL, par, leader, kBarW3)) goto w3_done;
            ptx::tc_fence_after();
            {
                uint32_t pk[64];  // the whole output row as bf16 pairs
                float2 ss2 = make_float2(0.f, 0.f);  // fused norm + gate: the row's sum of squares, in two parts
#pragma unroll
                for (int cb = 0; cb < 4; cb += 2) {
                    // two loads in flight per wait: O_FREE is on the path to the next block's first MMA
                    uint32_t a0[32], a1[32];
                    ptx::tmem_ld32(trow + kColO + 32 * cb, a0);
                    ptx::tmem_ld32(trow + kColO + 32 * cb + 32, a1);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const float x0 = __uint_as_float(a0[2 * u]) * f_o, x1 = __uint_as_float(a0[2 * u + 1]) * f_o;
                        const float y0 = __uint_as_float(a1[2 * u]) * f_o, y1 = __uint_as_float(a1[2 * u + 1]) * f_o;
                        pk[16 * cb + u] = ptx::pack_bf16(x0, x1);
                        pk[16 * cb + 16 + u] = ptx::pack_bf16(y0, y1);
                        if (kNormGate) {
                            ss2 = ptx::fma2(make_float2(x0, x1), make_float2(x0, x1), ss2);
                            ss2 = ptx::fma2(make_float2(y0, y1), make_float2(y0, y1), ss2);
                        }
                    }
                }
                ptx::tc_fence_before();
                ptx::named_bar_sync(kBarW3, 128);
                if (leader) arrive_leader(&c.bars[O_FREE]);
                uint8_t *erow = c.smem + kOffE + l * 128;
                const float rstd = kNormGate ? rsqrtf((ss2.x + ss2.y) * (1.f / kDim) + ng.eps) : 0.f;
                const float hr = 0.5f * rstd;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    if (kNormGate) {
                        // y = gamma o rstd sigmoid(g) on this half's 64 columns, written over the
                        // gate row in the staging tile, as a + a tanh(g/2) with a = (gamma rstd / 2) o,
                        // in paired fp32 operations (SFU tanh)
                        if (hh == 1 && leader) load_gate(t, 1);
                        if (!group_wait(c, G_FULL, (uint32_t)hh, leader, kBarW3)) goto w3_done;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            uint4 *slot = reinterpret_cast<uint4 *>(erow + ((ch ^ (l & 7)) << 4));
                            const uint4 g4 = *slot;
                            const float4 ga = *reinterpret_cast<const float4 *>(gsm + 64 * hh + 8 * ch);
                            const float4 gb = *reinterpret_cast<const float4 *>(gsm + 64 * hh + 8 * ch + 4);
                            const float gm[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                            const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
                            uint32_t yw[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const uint32_t w = pk[32 * hh + 4 * ch + e];
                                const float2 ga = mul2(make_float2(ptx::bf16_lo(gw[e]), ptx::bf16_hi(gw[e])),
                                                       make_float2(0.5f, 0.5f));
                                float th0, th1;
                                asm("tanh.approx.f32 %0, %1;" : "=f"(th0) : "f"(ga.x));
                                asm("tanh.approx.f32 %0, %1;" : "=f"(th1) : "f"(ga.y));
                                const float2 cg = mul2(make_float2(gm[2 * e], gm[2 * e + 1]), make_float2(hr, hr));
                                const float2 a = mul2(cg, make_float2(ptx::bf16_lo(w), ptx::bf16_hi(w)));
                                const float2 yv = ptx::fma2(a, make_float2(th0, th1), a);  // a (1 + tanh)
                                yw[e] = ptx::pack_bf16(yv.x, yv.y);
                            }
                            *slot = make_uint4(yw[0], yw[1], yw[2], yw[3]);
                        }
                    } else {
                        // the previous store must have finished reading the staging buffer
                        if (leader) ptx::bulk_wait_read();
                        ptx::named_bar_sync(kBarW3, 128);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch)
                            *reinterpret_cast<uint4 *>(erow + ((ch ^ (l & 7)) << 4)) =
                                make_uint4(pk[32 * hh + 4 * ch], pk[32 * hh + 4 * ch + 1], pk[32 * hh + 4 * ch + 2],
                                           pk[32 * hh + 4 * ch + 3]);
                    }
                    ptx::fence_proxy_async_smem();
                    ptx::named_bar_sync(kBarW3, 128);
                    if (leader) {
                        if (kNormGate)  // y is token-major: [batch][seq][heads][128]
                            ptx::tma_store_4d(&tm_o, c.smem + kOffE, 64 * hh, nh, tb(t) * kBlock + kRows * (int)rank,
                                              nb);
                        else
                            ptx::tma_store_3d(&tm_o, c.smem + kOffE, 64 * hh, tb(t) * kBlock + kRows * (int)rank, bh);
                        ptx::bulk_commit();
                    }
                }
            }
        }
    w3_done:;
        if (leader) {
            ptx::bulk_wait_all();  // output stores complete before the CTA exits
            // and the last gate load (if a wait for it was cut short): the k-th load
            // completes phase k, and the loads go one at a time
            if (kNormGate && g_issued > 0) {
                volatile int never = 0;
                ptx::mbar_wait(&c.bars[G_FULL], (uint32_t)(g_issued - 1) & 1u, &never);
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    cluster_sync();  // the even CTA's MMAs, which read this CTA's memory, are done
    if (warp == 2) {
        ptx::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(c.tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace pair

// The CTA-pair kernel covers bf16 inputs, head dim 128 and blocks of 256.
inline bool pair_supports(bool bf16, int dim, int block) { return bf16 && dim == 128 && block == 256; }

// Tensor map of a token-major output y [batch][seq][heads][128] (bf16), boxes of
// 64 channels of one head x 128 tokens (rows past seq are clipped on store).
inline bool make_token_major_map(CUtensorMap *map, void *y, int batch, int heads, int seq, std::string *err) {
    auto fn = tc::encode_fn(err);
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)pair::kDim, (cuuint64_t)heads, (cuuint64_t)seq, (cuuint64_t)batch};
    cuuint64_t strides[3] = {(cuuint64_t)pair::kDim * 2, (cuuint64_t)heads * pair::kDim * 2,
                             (cuuint64_t)seq * heads * pair::kDim * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)pair::kRows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, y, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = "cuTensorMapEncodeTiled (token-major output) failed (CUresult " + std::to_string((int)r) + ")";
        return false;
    }
    return true;
}

// Workspace of one CTA-pair prefill: the range guard's record per (batch, head), 48 bytes.
inline size_t pair_workspace_bytes(long long batch_heads) {
    return (size_t)batch_heads * sizeof(rg::RangeRec);
}

// ng != nullptr: the forward prefill with the normalisation and gating fused into
// its epilogue; o is then the token-major y. Two launches on `stream`: the plain
// kernel, which measures every (batch, head) into rec (pair_workspace_bytes of
// the caller's workspace), then pass 2, which recomputes the heads it flagged.
inline la_status launch_pair(const void *q, const void *k, const void *v, const float *slopes, int batch,
                             int heads, int seq, const float *state_in, void *o, float *state_out, Snapshots sn,
                             pair::PairPass pp, rg::RangeRec *rec,
                             cudaStream_t stream, std::string *err, const pair::PairNormGate *ng = nullptr) {
    const long long bh = (long long)batch * heads;
    if (ng && pp.anti) {
        *err = "the fused normalisation runs on the forward (causal) pass only";
        return LA_ERR_UNSUPPORTED;
    }
    if (!rec) {
        *err = "the CTA-pair prefill needs its workspace (the range guard's records)";
        return LA_ERR_INVALID_ARG;
    }
    CUtensorMap mq, mk, mv, mo, mg;
    if (!tc::make_map(&mq, q, seq, bh, err) || !tc::make_map(&mk, k, seq, bh, err) ||
        !tc::make_map(&mv, v, seq, bh, err) ||
        !(ng ? make_token_major_map(&mo, o, batch, heads, seq, err) : tc::make_map(&mo, o, seq, bh, err)))
        return LA_ERR_CUDA;
    if (ng) {
        if (!make_token_major_map(&mg, const_cast<__nv_bfloat16 *>(ng->gate), batch, heads, seq, err))
            return LA_ERR_CUDA;
    } else {
        mg = mo;  // unused
    }
    using Kernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                            const float *, int, int, const float *, float *, Snapshots, pair::PairPass,
                            pair::PairNormGate, rg::RangeRec *, const __nv_bfloat16 *, const __nv_bfloat16 *);
    const Kernel passes[2] = {
        ng ? pair::prefill_pair_kernel<false, true, false>
           : pp.anti ? pair::prefill_pair_kernel<true, false, false> : pair::prefill_pair_kernel<false, false, false>,
        ng ? pair::prefill_pair_kernel<false, true, true>
           : pp.anti ? pair::prefill_pair_kernel<true, false, true> : pair::prefill_pair_kernel<false, false, true>};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(bh * 2));
    cfg.blockDim = dim3(pair::kThreads);
    cfg.dynamicSmemBytes = pair::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // pass 2 is pass 1's programmatic dependent (it starts with griddepcontrol.wait)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    const pair::PairNormGate ngv = ng ? *ng : pair::PairNormGate{nullptr, nullptr, 0.f};
    for (int pass = 0; pass < 2; ++pass) {
        cfg.numAttrs = pass == 0 ? 1 : 2;
        cudaError_t e = cudaFuncSetAttribute(passes[pass], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)pair::kSmemBytes);
        if (e != cudaSuccess) {
            *err = std::string("cudaFuncSetAttribute(prefill_pair): ") + cudaGetErrorString(e);
            return LA_ERR_CUDA;
        }
        e = cudaLaunchKernelEx(&cfg, passes[pass], mq, mk, mv, mo, mg, slopes, heads, seq, state_in,
                               state_out, sn, pp, ngv, rec, static_cast<const __nv_bfloat16 *>(q),
                               static_cast<const __nv_bfloat16 *>(k));
        if (e != cudaSuccess) {
            *err = std::string("prefill_pair launch: ") + cudaGetErrorString(e);
            return LA_ERR_CUDA;
        }
    }
    err->clear();
    return LA_OK;
}

}  // namespace la
