// Prefill of the softmax attention layer that M1 places after every seven
// Lightning layers ("MINIMAX SIGNAL LAB · M1", §02: 64 query heads x 128,
// softmax K/V 8 x 128, RoPE on 64 of the 128 dims in the softmax layers only;
// §04: those layers keep a bf16 KV cache). Readings as for the decode step:
// grouped-query attention (query head h reads KV head h / (heads/kv_heads)),
// scores scaled by `scale`, rotate-half RoPE on the first `rot` dims, the
// cache holds rotated keys. `seq` new tokens of sequence b sit at positions
// start[b] .. start[b]+seq-1 (each sequence with its own cached prefix); token i
// attends causally to positions 0 .. start[b]+i:
//   o_i = sum_{p <= start[b]+i} softmax_p(scale * rope(q_i) . k_p) v_p.
//
// Two kernels:
//   gqp_rope_kernel     one CTA per (token, sequence): the token's angles once
//                       (double), then q rotated into a bf16 workspace and the
//                       rotated key and the value written into the cache.
//   gqp_attn_kernel     causal softmax attention on the tensor cores (tcgen05,
//                       TMEM accumulators, TMA-fed), one CTA per 256 query rows
//                       of one query head, as two 128-row tiles t = 0, 1.
//
// Attention, per key tile j of 128 positions (K_j, V_j from the cache):
//   S_t = Q_t K_j^T         SS MMA bf16, M128 N128 K128 -> TMEM (fp32)
//   softmax warpgroup t:    row max, P_t = 2^(S_t * scale * log2 e - m) as bf16
//                           written over the first 64 columns of S_t in TMEM
//                           (the row sum l adds the fp32 weights);
//                           the running max m is raised only when a row's max
//                           grows by more than 2^8, and O_t is then rescaled
//                           in TMEM before the next P V (P stays <= 2^8)
//   O_t += P_t V_j          TS MMA bf16 (A = P from TMEM), M128 N128 K128, in two
//                           halves of 64 keys, each as soon as its half of P is written
// The MMA thread issues PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), ... so each
// tile's softmax overlaps the other tile's MMAs. MMAs issued by one thread run
// in order, so QK_t(j+1) writes S_t only after PV_t(j) has read P_t, and the
// commit that announces S_t(j+1) also covers PV_t(j) (O_t is complete when the
// softmax warpgroup reads it). The epilogue scales O_t by 1/l, rounds it to
// bf16 into the Q_t tile's shared memory and stores it with TMA.
// CTAs go KV head by KV head (query head fastest, then the query rows from the longest
// down), so the CTAs resident at a time read one KV head's keys and values, which L2 holds
// (67 MB at 131072 positions); heavy-first within a KV head keeps the tail short.
// A query tile reads the key tiles up to its last row's position. Only the
// last of them can reach past position start[b]+seq-1, into cache rows this
// call neither wrote nor was given: their scores are masked, and their value
// rows are zeroed in shared memory before P V (a masked weight is 0, but
// 0 x NaN is NaN).
//
// Warp roles: warp 0 TMA, warp 1 MMA (the whole warp follows the waits, one elected lane
// issues), warp 2 TMEM, warps 4-7 and 8-11 the softmax warpgroups of tiles 0 and 1; the
// control warps hand most of their registers to the softmax warps. Every wait is bounded.
// Shared memory: Q_0, Q_1 (32 KB each, also the output staging), 2 stages of
// K and of V (32 KB each), barriers. TMEM: [0,128) S_0/P_0, [128,256) S_1/P_1,
// [256,384) O_0, [384,512) O_1.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <string>

#include "common.cuh"
#include "prefill_tc.cuh"
#include "tc_ptx.cuh"

namespace la {
namespace gqp {

constexpr int kThreads = 384;
constexpr int kDim = 128;
constexpr int kRows = 128;                       // query rows per tile, positions per key tile
constexpr int kQRows = 2 * kRows;                // query rows per CTA
constexpr uint32_t kBoxBytes = 16384;            // 128 rows x 64 bf16 (128-byte rows)
constexpr uint32_t kTileBytes = 2 * kBoxBytes;   // 128 rows x 128 dims
constexpr int kStages = 2;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
constexpr int kNumBars = 18;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;  // + slack to align the base to 1024

// registers per thread after the split: the control warpgroup gives its share to the two
// softmax warpgroups. The launcher checks the kernel's allocation (threads x registers) holds
// the split, since a setmaxnreg.inc beyond it would wait forever.
constexpr int kCtrlRegs = 80, kSoftmaxRegs = 200;
constexpr int kSplitRegs = 4 * 32 * kCtrlRegs + 8 * 32 * kSoftmaxRegs;
static_assert(kSplitRegs <= kThreads * ((65536 / kThreads) & ~7), "register split above the launch's");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;       // + 128 t

constexpr int Q_FULL = 0, K_FULL = 1 /* 2 */, K_EMPTY = 3 /* 2 */, V_FULL = 5 /* 2 */, V_EMPTY = 7 /* 2 */,
              S_FULL = 9 /* 2 */, P_FULL = 11 /* 2 x 2: tile, half */, O_FINAL = 15 /* 2 */, DRAIN = 17;

// the running max is raised only past this margin (log2 units): P <= 2^8
constexpr float kRescaleMargin = 8.f;
constexpr float kLog2eF = 1.4426950408889634f;

__host__ __device__ constexpr uint32_t idesc(int M, int N, uint32_t fmt, bool a_mn, bool b_mn) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescQK = idesc(128, 128, 1, false, false);  // Q (K-major) x K (K-major), bf16
constexpr uint32_t kIdescPV = idesc(128, 128, 1, false, true);   // P (TMEM) x V (MN-major), bf16

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// --------------------------------------------------------------------- RoPE

// grid (seq, batch), 256 threads. q_rot[b][h][i] = rope(q[b][h][i], start[b]+i);
// k_cache[b][g][start[b]+i] = rope(k_new[b][g][i], start[b]+i); v_cache[..] = v_new.
// A start[b] outside 0 .. cap-seq skips sequence b and is reported in the status word.
// Elements travel in pairs (rot % 4 == 0 keeps a pair on one side of the
// rotation); angles in double, rotation in fp32, results rounded to bf16.
__global__ void __launch_bounds__(256)
gqp_rope_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k_new,
                const __nv_bfloat16 *__restrict__ v_new, __nv_bfloat16 *__restrict__ k_cache,
                __nv_bfloat16 *__restrict__ v_cache, __nv_bfloat16 *__restrict__ q_rot, int heads, int kv_heads,
                int seq, const int *__restrict__ start, int cap, int rot, double base) {
    __shared__ float cs[kDim / 2], sn[kDim / 2];
    const int i = blockIdx.x, b = blockIdx.y, st = start[b], half = rot / 2;
    if (st < 0 || st > cap - seq) {
        if (i == 0 && threadIdx.x == 0) atomicOr(&g_device_status, kBadDeviceArgFlag);
        return;
    }
    const int pos = st + i;
    for (int c = threadIdx.x; c < half; c += blockDim.x) {
        double s, co;
        sincos((double)pos * pow(base, -2.0 * c / (double)rot), &s, &co);
        cs[c] = (float)co;
        sn[c] = (float)s;
    }
    __syncthreads();
    constexpr int kPairs = kDim / 2;
    const int rows = heads + 2 * kv_heads;
    for (int u = threadIdx.x; u < rows * kPairs; u += blockDim.x) {
        const int hr = u / kPairs, c = 2 * (u - hr * kPairs);
        const uint32_t *src;
        uint32_t *dst;
        if (hr < heads) {
            const size_t row = ((size_t)b * heads + hr) * seq + i;
            src = reinterpret_cast<const uint32_t *>(q + row * kDim);
            dst = reinterpret_cast<uint32_t *>(q_rot + row * kDim);
        } else if (hr < heads + kv_heads) {
            const size_t g = (size_t)b * kv_heads + (hr - heads);
            src = reinterpret_cast<const uint32_t *>(k_new + (g * seq + i) * kDim);
            dst = reinterpret_cast<uint32_t *>(k_cache + (g * cap + pos) * kDim);
        } else {
            const size_t g = (size_t)b * kv_heads + (hr - heads - kv_heads);
            reinterpret_cast<uint32_t *>(v_cache + (g * cap + pos) * kDim)[c / 2] =
                reinterpret_cast<const uint32_t *>(v_new + (g * seq + i) * kDim)[c / 2];
            continue;
        }
        const uint32_t x = src[c / 2];
        if (c >= rot) {
            dst[c / 2] = x;
            continue;
        }
        const bool lo = c < half;
        const int a = lo ? c : c - half;  // angle index of this pair's first element
        const uint32_t y = src[(lo ? c + half : c - half) / 2];
        const float sg = lo ? -1.f : 1.f;
        const float r0 = fmaf(sg * ptx::bf16_lo(y), sn[a], ptx::bf16_lo(x) * cs[a]);
        const float r1 = fmaf(sg * ptx::bf16_hi(y), sn[a + 1], ptx::bf16_hi(x) * cs[a + 1]);
        dst[c / 2] = ptx::pack_bf16(r0, r1);
    }
}

// ---------------------------------------------------------------- attention

// 32 lanes x 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 128 consecutive 32-bit columns (four x32 loads, one wait by the caller)
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
#define GQP_LD32(Q)                                                                                        \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                 \
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                                 \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                \
                 : "=r"(r[32 * Q + 0]), "=r"(r[32 * Q + 1]), "=r"(r[32 * Q + 2]), "=r"(r[32 * Q + 3]),     \
                   "=r"(r[32 * Q + 4]), "=r"(r[32 * Q + 5]), "=r"(r[32 * Q + 6]), "=r"(r[32 * Q + 7]),     \
                   "=r"(r[32 * Q + 8]), "=r"(r[32 * Q + 9]), "=r"(r[32 * Q + 10]), "=r"(r[32 * Q + 11]),   \
                   "=r"(r[32 * Q + 12]), "=r"(r[32 * Q + 13]), "=r"(r[32 * Q + 14]), "=r"(r[32 * Q + 15]), \
                   "=r"(r[32 * Q + 16]), "=r"(r[32 * Q + 17]), "=r"(r[32 * Q + 18]), "=r"(r[32 * Q + 19]), \
                   "=r"(r[32 * Q + 20]), "=r"(r[32 * Q + 21]), "=r"(r[32 * Q + 22]), "=r"(r[32 * Q + 23]), \
                   "=r"(r[32 * Q + 24]), "=r"(r[32 * Q + 25]), "=r"(r[32 * Q + 26]), "=r"(r[32 * Q + 27]), \
                   "=r"(r[32 * Q + 28]), "=r"(r[32 * Q + 29]), "=r"(r[32 * Q + 30]), "=r"(r[32 * Q + 31])  \
                 : "r"(taddr + 32u * Q)                                                                    \
                 : "memory")
    GQP_LD32(0);
    GQP_LD32(1);
    GQP_LD32(2);
    GQP_LD32(3);
#undef GQP_LD32
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

using ptx::fma2;

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// P = 2^(S sl2 - m) for keys 64 H .. 64 H + 63 of one row of scores: bf16 pairs into TMEM
// columns [taddr + 32 H, taddr + 32 H + 32); returns the sum of the fp32 weights (summing
// the bf16-rounded ones instead keeps o an exact weighted mean but cost 4-5 %).
template <int H>
__device__ __forceinline__ float p_half(const uint32_t (&v)[128], float sl2, float m, uint32_t taddr) {
    const float2 sl = make_float2(sl2, sl2), nm = make_float2(-m, -m), one = make_float2(1.f, 1.f);
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 2 * H; q < 2 * H + 2; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const float2 x = fma2(make_float2(__uint_as_float(v[32 * q + 2 * u]), __uint_as_float(v[32 * q + 2 * u + 1])),
                                  sl, nm);
            const float2 p = make_float2(ptx::ex2(x.x), ptx::ex2(x.y));
            pk[u] = ptx::pack_bf16(p.x, p.y);
            acc = fma2(p, one, acc);
        }
        ptx::tmem_st16(taddr + 16u * q, pk);
    }
    return acc.x + acc.y;
}

// one lane of a converged warp (the lowest active one)
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(pred));
    return pred != 0;
}

// Work of one CTA: query rows i0 .. i0+255 of head h of sequence b.
struct Work {
    int bh, bkv, i0, n[2];  // n[t]: key tiles that query tile t reads (0: tile absent)
};

__device__ __forceinline__ Work work_of(int heads, int kv_heads, int batch, int seq, const int *start,
                                        int *start_b) {
    const int group = heads / kv_heads;
    const int npairs = (seq + kQRows - 1) / kQRows;
    const int x = blockIdx.x;
    const int hq = x % group, rest = x / group;
    const int pi = npairs - 1 - rest % npairs;  // the longest rows first, within a KV head
    const int bkv = rest / npairs;
    const int b = bkv / kv_heads, g = bkv - b * kv_heads;
    Work w;
    w.bh = b * heads + g * group + hq;
    w.bkv = bkv;
    w.i0 = kQRows * pi;
    *start_b = start[b];
    const int st = *start_b;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int r0 = w.i0 + kRows * t;
        w.n[t] = r0 < seq ? (st + min(r0 + kRows - 1, seq - 1)) / kRows + 1 : 0;
    }
    return w;
}

// tm_q: q_rot [batch*heads][seq][128]; tm_k, tm_v: caches [batch*kv_heads][cap][128];
// tm_o: o [batch*heads][seq][128]. All 128-byte swizzled boxes of 64 x 128. Sequence b
// reads cache rows 0 .. start[b]+seq-1 only: its last key tile may reach past them, and
// those value rows are zeroed in shared memory before P V (their weights are 0, but the
// rows may hold anything, and 0 x NaN is NaN); the scores of those keys are masked.
__global__ void __launch_bounds__(kThreads, 1)
gqp_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, int batch,
                int heads, int kv_heads, int seq, const int *__restrict__ start, int cap, float sl2) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_addr(smem_raw);
    const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
    Ctx c;
    c.smem = smem_raw + pad;
    c.sbase = raw_addr + pad;
    c.bars = reinterpret_cast<uint64_t *>(c.smem + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c.smem + kOffMisc);
    c.abort = reinterpret_cast<volatile int *>(c.smem + kOffMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int st = 0;  // this sequence's start
    const Work w = work_of(heads, kv_heads, batch, seq, start, &st);
    if (st < 0 || st > cap - seq) return;  // reported by the RoPE launch; nothing allocated yet
    const int nmax = max(w.n[0], w.n[1]);
    const int kend = st + seq;  // cache rows 0 .. kend-1 hold this sequence's keys

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) ptx::mbar_init(&c.bars[i], 1);
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&c.bars[P_FULL + i], 4);  // one arrival per softmax warp
        *c.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_o);
    }
    if (warp == 2) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    c.tmem = *tmem_slot;

    // registers: the control warps (TMA, MMA, TMEM) give theirs to the softmax warps
    // (4 x 32 x 56 + 8 x 32 x 224 = 384 x 168, the launch's allocation)
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                bool ok = true;
                uint64_t *qbar = &c.bars[Q_FULL];
                ptx::mbar_arrive_expect_tx(qbar, (w.n[1] > 0 ? 2 : 1) * kTileBytes);
                for (int t = 0; t < 2; ++t) {
                    if (w.n[t] == 0) continue;
                    uint8_t *dst = c.smem + kOffQ + t * kTileBytes;
                    ptx::tma_load_3d(dst, &tm_q, qbar, 0, w.i0 + kRows * t, w.bh);
                    ptx::tma_load_3d(dst + kBoxBytes, &tm_q, qbar, 64, w.i0 + kRows * t, w.bh);
                }
                int k_issued = 0, v_issued = 0;
                for (int j = 0; j < nmax && ok; ++j) {
                    const int st = j & 1;
                    const uint32_t epar = ((uint32_t)(j >> 1) & 1u) ^ 1u;  // phase of the stage's previous use
                    if (j >= kStages && !wait_bar(c, K_EMPTY + st, epar)) { ok = false; break; }
                    uint64_t *kb = &c.bars[K_FULL + st];
                    uint8_t *kd = c.smem + kOffK + st * kTileBytes;
                    ptx::mbar_arrive_expect_tx(kb, kTileBytes);
                    ptx::tma_load_3d(kd, &tm_k, kb, 0, kRows * j, w.bkv);
                    ptx::tma_load_3d(kd + kBoxBytes, &tm_k, kb, 64, kRows * j, w.bkv);
                    k_issued = j + 1;
                    if (j >= kStages && !wait_bar(c, V_EMPTY + st, epar)) { ok = false; break; }
                    uint64_t *vb = &c.bars[V_FULL + st];
                    uint8_t *vd = c.smem + kOffV + st * kTileBytes;
                    ptx::mbar_arrive_expect_tx(vb, kTileBytes);
                    ptx::tma_load_3d(vd, &tm_v, vb, 0, kRows * j, w.bkv);
                    ptx::tma_load_3d(vd + kBoxBytes, &tm_v, vb, 64, kRows * j, w.bkv);
                    v_issued = j + 1;
                }
                // let every copy issued land before the CTA may exit (earlier ones were consumed)
                volatile int never = 0;
                ptx::mbar_wait(qbar, 0, &never);
                for (int j = k_issued > kStages ? k_issued - kStages : 0; j < k_issued; ++j)
                    ptx::mbar_wait(&c.bars[K_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, &never);
                for (int j = v_issued > kStages ? v_issued - kStages : 0; j < v_issued; ++j)
                    ptx::mbar_wait(&c.bars[V_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, &never);
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            // the whole warp follows the waits; one elected lane issues the MMAs and commits
            {
                const uint32_t tm = c.tmem;
                const uint64_t dq0 = sdesc(c.sbase + kOffQ, 16u, 1024u);
                const uint64_t dk0 = sdesc(c.sbase + kOffK, 16u, 1024u);
                const uint64_t dv0 = sdesc(c.sbase + kOffV, kBoxBytes, 1024u);
                int k_ready = -1, v_ready = -1;
                bool ok = wait_bar(c, Q_FULL, 0);
                if (ok) ptx::tc_fence_after();
                // S_t = Q_t K_j^T
                auto qk = [&](int t, int j) -> bool {
                    if (j > k_ready) {
                        if (!wait_bar(c, K_FULL + (j & 1), (uint32_t)(j >> 1) & 1u)) return false;
                        ptx::tc_fence_after();
                        k_ready = j;
                    }
                    const uint64_t dq = dq0 + (uint64_t)((t * kTileBytes) >> 4);
                    const uint64_t dk = dk0 + (uint64_t)(((j & 1) * kTileBytes) >> 4);
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint64_t koff = (uint64_t)(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4);
                            ptx::mma_ss(tm + kColS + 128u * t, dq + koff, dk + koff, kIdescQK, k > 0);
                        }
                        ptx::mma_commit(&c.bars[S_FULL + t]);
                        if (t == 1 || j >= w.n[1]) ptx::mma_commit(&c.bars[K_EMPTY + (j & 1)]);  // last reader of K_j
                    }
                    __syncwarp();
                    return true;
                };
                // O_t += P_t V_j
                auto pv = [&](int t, int j) -> bool {
                    if (j > v_ready) {
                        if (!wait_bar(c, V_FULL + (j & 1), (uint32_t)(j >> 1) & 1u)) return false;
                        v_ready = j;
                        const int live = kend - kRows * j;  // rows of this value tile inside the sequence
                        if (live < kRows) {
                            // the rows past the sequence: zeros, as the whole warp stores them
                            uint8_t *vd = c.smem + kOffV + (j & 1) * kTileBytes;
                            for (int u = lane; u < (kRows - live) * 16; u += 32) {
                                const int row = live + (u >> 4), box = (u >> 3) & 1, ch = u & 7;
                                *reinterpret_cast<uint4 *>(vd + box * kBoxBytes + row * 128 + ch * 16) =
                                    make_uint4(0u, 0u, 0u, 0u);
                            }
                            ptx::fence_proxy_async_smem();
                            __syncwarp();
                        }
                    }
                    const uint64_t dv = dv0 + (uint64_t)(((j & 1) * kTileBytes) >> 4);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        // keys 64 hh .. 64 hh + 63, as soon as their half of P is in TMEM
                        if (!wait_bar(c, P_FULL + 2 * t + hh, (uint32_t)j & 1u)) return false;
                        ptx::tc_fence_after();
                        if (elect_one()) {
#pragma unroll
                            for (int k = 4 * hh; k < 4 * hh + 4; ++k)
                                ptx::mma_ts(tm + kColO + 128u * t, tm + kColS + 128u * t + 8u * k,
                                            dv + (uint64_t)(k * (2048 >> 4)), kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
                            if (hh == 1) {
                                if (t == 1 || j >= w.n[1]) ptx::mma_commit(&c.bars[V_EMPTY + (j & 1)]);  // last reader of V_j
                                if (j == w.n[t] - 1) ptx::mma_commit(&c.bars[O_FINAL + t]);
                            }
                        }
                        __syncwarp();
                    }
                    return true;
                };
                for (int t = 0; t < 2 && ok; ++t)
                    if (w.n[t] > 0) ok = qk(t, 0);
                for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll 1
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (j >= w.n[t]) continue;
                        ok = pv(t, j);
                        if (ok && j + 1 < w.n[t]) ok = qk(t, j + 1);
                    }
                }
                if (elect_one()) ptx::mma_commit(&c.bars[DRAIN]);
                __syncwarp();
                volatile int never = 0;
                ptx::mbar_wait(&c.bars[DRAIN], 0, &never);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ------------------------------------------------------------ softmax warpgroups
        const int t = (warp - 4) >> 2;             // query tile
        const int r = threadIdx.x & 127;           // TMEM lane = row of the tile
        const bool leader = r == 0;
        const int bar_id = 1 + t;
        const uint32_t trow = c.tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint32_t cs_ = kColS + 128u * t, co_ = kColO + 128u * t;
        const int nt = w.n[t];
        const int pmin = st + w.i0 + kRows * t;     // position of the tile's first row
        const int qpos = pmin + r;
        float m = -INFINITY, l = 0.f;               // running max (log2 units) and sum
        bool done = nt > 0;
        for (int j = 0; j < nt; ++j) {
            // every thread waits itself: the lanes of a warp poll together and agree
            if (!ptx::mbar_wait(&c.bars[S_FULL + t], (uint32_t)j & 1u, c.abort)) { done = false; break; }
            ptx::tc_fence_after();
            uint32_t v[128];
            tmem_ld128(trow + cs_, v);
            ptx::tmem_ld_wait();
            const bool masked = kRows * j + kRows - 1 > pmin;  // the tile reaches past some row's position
            if (masked) {
                const int lim = qpos - kRows * j;   // last live column of this row
#pragma unroll
                for (int u = 0; u < 128; ++u)
                    if (u > lim) v[u] = 0xff800000u;  // -inf
            }
            float mx0 = __uint_as_float(v[0]), mx1 = __uint_as_float(v[1]);
#pragma unroll
            for (int u = 2; u < 126; u += 4) {
                mx0 = max3(mx0, __uint_as_float(v[u]), __uint_as_float(v[u + 1]));
                mx1 = max3(mx1, __uint_as_float(v[u + 2]), __uint_as_float(v[u + 3]));
            }
            const float mnew = fmaxf(m, max3(mx0, mx1, fmaxf(__uint_as_float(v[126]), __uint_as_float(v[127]))) * sl2);
            // raise the running max (warp-uniformly: the TMEM accesses are collective)
            const bool raise = __any_sync(0xffffffffu, mnew > m + kRescaleMargin);
            float alpha = 1.f;
            if (raise) {
                alpha = ptx::ex2(m - mnew);   // 0 on the first tile
                l *= alpha;
                m = mnew;
            }
            // P = 2^(S sl2 - m) as bf16 pairs over the first 64 columns of S, in two halves of
            // 64 keys: the P V of the first half runs while the second is computed
            if (!raise || j == 0) {
                l += p_half<0>(v, sl2, m, trow + cs_);
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&c.bars[P_FULL + 2 * t]);
                l += p_half<1>(v, sl2, m, trow + cs_);
            } else {
                // O is rescaled once the scores are no longer needed, before either half of P V
                l += p_half<0>(v, sl2, m, trow + cs_);
                l += p_half<1>(v, sl2, m, trow + cs_);
#pragma unroll 1
                for (int q = 0; q < 8; ++q) {
                    uint32_t a[16];
                    tmem_ld16(trow + co_ + 16u * q, a);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; ++u) a[u] = __float_as_uint(__uint_as_float(a[u]) * alpha);
                    ptx::tmem_st16(trow + co_ + 16u * q, a);
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&c.bars[P_FULL + 2 * t]);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&c.bars[P_FULL + 2 * t + 1]);
        }
        if (done) done = ptx::mbar_wait(&c.bars[O_FINAL + t], 0, c.abort);
        done = ptx::named_bar_and(bar_id, 128, done);  // the four warps agree before the epilogue
        if (done) {
            // O / l -> bf16 -> this tile's Q buffer (128B-swizzled, as TMA reads it) -> TMA store;
            // rows past seq are clipped by the store
            ptx::tc_fence_after();
            const float inv = 1.f / l;
            uint8_t *tile = c.smem + kOffQ + t * kTileBytes;
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                uint32_t a0[32], a1[32];
                ptx::tmem_ld32(trow + co_ + 64u * hb, a0);
                ptx::tmem_ld32(trow + co_ + 64u * hb + 32u, a1);
                ptx::tmem_ld_wait();
                uint8_t *row = tile + hb * kBoxBytes + r * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint32_t *x = ch < 4 ? &a0[8 * ch] : &a1[8 * (ch - 4)];
                    uint32_t pk[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        pk[u] = ptx::pack_bf16(__uint_as_float(x[2 * u]) * inv, __uint_as_float(x[2 * u + 1]) * inv);
                    *reinterpret_cast<uint4 *>(row + ((ch ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::named_bar_sync(bar_id, 128);
            if (leader) {
                ptx::tma_store_3d(&tm_o, tile, 0, w.i0 + kRows * t, w.bh);
                ptx::tma_store_3d(&tm_o, tile + kBoxBytes, 64, w.i0 + kRows * t, w.bh);
                ptx::bulk_commit();
                ptx::bulk_wait_all();  // output stores complete before the CTA exits
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(c.tmem, kTmemCols);
    }
}

}  // namespace gqp

// [outer][rows][128] bf16 with `stride_rows` rows between consecutive outer
// indices (rows <= stride_rows), as a 3-D tensor map of 64 x 128 boxes with
// the 128-byte swizzle; rows past `rows` read as zeros and are clipped on store.
inline bool gqp_make_map(CUtensorMap *map, const void *base, long long rows, long long stride_rows,
                         long long outer, std::string *err) {
    auto fn = tc::encode_fn(err);
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)gqp::kDim, (cuuint64_t)rows, (cuuint64_t)outer};
    cuuint64_t strides[2] = {(cuuint64_t)gqp::kDim * 2, (cuuint64_t)stride_rows * gqp::kDim * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)gqp::kRows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = "cuTensorMapEncodeTiled failed (CUresult " + std::to_string((int)r) + ")";
        return false;
    }
    return true;
}

// q, o: [batch][heads][seq][128]; k_new, v_new: [batch][kv_heads][seq][128];
// caches [batch][kv_heads][cap][128]; q_rot: workspace of q's size. bf16 throughout.
inline la_status launch_gqa_prefill(const void *q, const void *k_new, const void *v_new, void *k_cache,
                                    void *v_cache, const int *start, int batch, int heads, int kv_heads, int seq, int cap,
                                    int rot, double base, float scale, void *o, void *q_rot, cudaStream_t stream,
                                    std::string *err) {
    using bf = __nv_bfloat16;
    gqp::gqp_rope_kernel<<<dim3((unsigned)seq, (unsigned)batch), 256, 0, stream>>>(
        static_cast<const bf *>(q), static_cast<const bf *>(k_new), static_cast<const bf *>(v_new),
        static_cast<bf *>(k_cache), static_cast<bf *>(v_cache), static_cast<bf *>(q_rot), heads, kv_heads, seq,
        start, cap, rot, base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *err = std::string("gqa prefill rope launch: ") + cudaGetErrorString(e);
        return LA_ERR_CUDA;
    }
    const long long bh = (long long)batch * heads, bkv = (long long)batch * kv_heads;
    CUtensorMap mq, mk, mv, mo;
    if (!gqp_make_map(&mq, q_rot, seq, seq, bh, err) || !gqp_make_map(&mk, k_cache, cap, cap, bkv, err) ||
        !gqp_make_map(&mv, v_cache, cap, cap, bkv, err) || !gqp_make_map(&mo, o, seq, seq, bh, err))
        return LA_ERR_CUDA;
    e = cudaFuncSetAttribute(gqp::gqp_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gqp::kSmemBytes);
    if (e != cudaSuccess) {
        *err = std::string("cudaFuncSetAttribute(gqa prefill attention): ") + cudaGetErrorString(e);
        return LA_ERR_CUDA;
    }
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, gqp::gqp_attn_kernel);
    if (e != cudaSuccess || fa.numRegs * gqp::kThreads < gqp::kSplitRegs) {
        // the warps' register split would wait for registers the launch never holds
        *err = "gqa prefill attention: register allocation below the kernel's split";
        return LA_ERR_CUDA;
    }
    const long long ctas = bh * ((seq + gqp::kQRows - 1) / gqp::kQRows);
    gqp::gqp_attn_kernel<<<(unsigned)ctas, gqp::kThreads, gqp::kSmemBytes, stream>>>(
        mq, mk, mv, mo, batch, heads, kv_heads, seq, start, cap, scale * gqp::kLog2eF);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        *err = std::string("gqa prefill attention launch: ") + cudaGetErrorString(e);
        return LA_ERR_CUDA;
    }
    err->clear();
    return LA_OK;
}

}  // namespace la

// ------------------------------------------------------------------ float32 path (CUDA cores)
namespace la {
namespace gqs {

constexpr int kThreads = 128;
constexpr int kQRows = 16;   // query rows per CTA (8 threads per row)
constexpr int kKeys = 64;    // keys per tile
constexpr int kDim = 128;
constexpr int kKPitch = kDim + 1;  // padded key rows: the 8 threads of a row read 8 different banks
constexpr uint32_t kSmemBytes = (kQRows * kDim + kKeys * kKPitch + kKeys * kDim + kQRows * kKeys) * 4;

// grid (seq, batch), 256 threads: q_rot = rope(q), cache rows start[b]+i <- rope(k_new), v_new.
// float32 throughout; angles in double. A start[b] outside 0 .. cap-seq skips sequence b and is
// reported in the status word.
__global__ void __launch_bounds__(256)
gqs_rope_kernel(const float *__restrict__ q, const float *__restrict__ k_new, const float *__restrict__ v_new,
                float *__restrict__ k_cache, float *__restrict__ v_cache, float *__restrict__ q_rot, int heads,
                int kv_heads, int seq, const int *__restrict__ start, int cap, int rot, double base) {
    __shared__ float cs[kDim / 2], sn[kDim / 2];
    const int i = blockIdx.x, b = blockIdx.y, st = start[b], half = rot / 2;
    if (st < 0 || st > cap - seq) {
        if (i == 0 && threadIdx.x == 0) atomicOr(&g_device_status, kBadDeviceArgFlag);
        return;
    }
    const int pos = st + i;
    for (int c = threadIdx.x; c < half; c += blockDim.x) {
        double s, co;
        sincos((double)pos * pow(base, -2.0 * c / (double)rot), &s, &co);
        cs[c] = (float)co;
        sn[c] = (float)s;
    }
    __syncthreads();
    const int rows = heads + 2 * kv_heads;
    for (int u = threadIdx.x; u < rows * kDim; u += blockDim.x) {
        const int hr = u / kDim, c = u - hr * kDim;
        const float *src;
        float *dst;
        if (hr < heads) {
            const size_t row = ((size_t)b * heads + hr) * seq + i;
            src = q + row * kDim;
            dst = q_rot + row * kDim;
        } else if (hr < heads + kv_heads) {
            const size_t g = (size_t)b * kv_heads + (hr - heads);
            src = k_new + (g * seq + i) * kDim;
            dst = k_cache + (g * cap + pos) * kDim;
        } else {
            const size_t g = (size_t)b * kv_heads + (hr - heads - kv_heads);
            v_cache[(g * cap + pos) * kDim + c] = v_new[(g * seq + i) * kDim + c];
            continue;
        }
        if (c >= rot) {
            dst[c] = src[c];
        } else if (c < half) {
            dst[c] = fmaf(-src[c + half], sn[c], src[c] * cs[c]);
        } else {
            dst[c] = fmaf(src[c - half], sn[c - half], src[c] * cs[c - half]);
        }
    }
}

// grid (ceil(seq / 16), heads, batch), 128 threads; dynamic shared memory kSmemBytes.
// Thread t takes row r = t / 8 of the CTA's 16 query rows: scores for keys t%8, t%8 + 8, ...
// of each 64-key tile, then output dims 16 (t%8) .. 16 (t%8) + 15. Exact online softmax in
// fp32 (the running max is raised on every increase); keys past start[b]+seq are never read.
__global__ void __launch_bounds__(kThreads)
gqs_attn_kernel(const float *__restrict__ q_rot, const float *__restrict__ k_cache, const float *__restrict__ v_cache,
                float *__restrict__ o, int heads, int kv_heads, int seq, const int *__restrict__ start, int cap,
                float scale) {
    extern __shared__ float sm[];
    float *qs = sm, *ks = qs + kQRows * kDim, *vs = ks + kKeys * kKPitch, *ps = vs + kKeys * kDim;
    const int i0 = blockIdx.x * kQRows, h = blockIdx.y, b = blockIdx.z;
    const int group = heads / kv_heads;
    const size_t bh = (size_t)b * heads + h, kv = (size_t)b * kv_heads + h / group;
    const int t = threadIdx.x, r = t >> 3, j8 = t & 7;
    const int st = start[b];
    if (st < 0 || st > cap - seq) return;  // reported by the RoPE launch
    const int qpos = st + i0 + r;                    // this row's position
    const int kend = min(st + i0 + kQRows, st + seq);  // keys 0 .. kend-1 are needed
    for (int e = t; e < kQRows * kDim; e += kThreads) {
        const int rr = e / kDim;
        qs[e] = i0 + rr < seq ? q_rot[(bh * seq + i0 + rr) * kDim + e % kDim] : 0.f;
    }
    float m = -INFINITY, l = 0.f, acc[16];
#pragma unroll
    for (int d = 0; d < 16; ++d) acc[d] = 0.f;
    for (int k0 = 0; k0 < kend; k0 += kKeys) {
        __syncthreads();  // the previous tile's keys, values and weights are no longer read
        for (int e = t; e < kKeys * kDim; e += kThreads) {
            const int kk = e / kDim, c = e % kDim;
            const bool live = k0 + kk < kend;
            ks[kk * kKPitch + c] = live ? k_cache[(kv * cap + k0 + kk) * kDim + c] : 0.f;
            vs[kk * kDim + c] = live ? v_cache[(kv * cap + k0 + kk) * kDim + c] : 0.f;
        }
        __syncthreads();
        float sc[8];
        float mt = -INFINITY;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int kk = j8 + 8 * u;
            float dot = 0.f;
#pragma unroll 8
            for (int c = 0; c < kDim; ++c) dot = fmaf(qs[r * kDim + c], ks[kk * kKPitch + c], dot);
            sc[u] = (k0 + kk <= qpos && k0 + kk < kend) ? dot * scale : -INFINITY;
            mt = fmaxf(mt, sc[u]);
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float mnew = fmaxf(m, mt);
        const float alpha = mnew == -INFINITY ? 1.f : __expf(m - mnew);  // 0 on a row's first live tile
        float ls = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float p = sc[u] == -INFINITY ? 0.f : __expf(sc[u] - mnew);
            ps[r * kKeys + j8 + 8 * u] = p;
            ls += p;
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        l = l * alpha + ls;
        m = mnew;
        __syncwarp();
#pragma unroll
        for (int d = 0; d < 16; ++d) acc[d] *= alpha;
        for (int kk = 0; kk < kKeys; ++kk) {
            const float p = ps[r * kKeys + kk];
            const float *vrow = vs + kk * kDim + 16 * j8;
#pragma unroll
            for (int d = 0; d < 16; ++d) acc[d] = fmaf(p, vrow[d], acc[d]);
        }
    }
    if (i0 + r < seq) {
        const float inv = 1.f / l;
        float *dst = o + (bh * seq + i0 + r) * kDim + 16 * j8;
#pragma unroll
        for (int d = 0; d < 16; ++d) dst[d] = acc[d] * inv;
    }
}

}  // namespace gqs

inline la_status launch_gqa_prefill_f32(const void *q, const void *k_new, const void *v_new, void *k_cache,
                                        void *v_cache, const int *start, int batch, int heads, int kv_heads, int seq,
                                        int cap, int rot, double base, float scale, void *o, void *q_rot,
                                        cudaStream_t stream, std::string *err) {
    gqs::gqs_rope_kernel<<<dim3((unsigned)seq, (unsigned)batch), 256, 0, stream>>>(
        static_cast<const float *>(q), static_cast<const float *>(k_new), static_cast<const float *>(v_new),
        static_cast<float *>(k_cache), static_cast<float *>(v_cache), static_cast<float *>(q_rot), heads, kv_heads,
        seq, start, cap, rot, base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *err = std::string("gqa prefill rope launch: ") + cudaGetErrorString(e);
        return LA_ERR_CUDA;
    }
    e = cudaFuncSetAttribute(gqs::gqs_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gqs::kSmemBytes);
    if (e != cudaSuccess) {
        *err = std::string("cudaFuncSetAttribute(gqa prefill f32): ") + cudaGetErrorString(e);
        return LA_ERR_CUDA;
    }
    gqs::gqs_attn_kernel<<<dim3((unsigned)((seq + gqs::kQRows - 1) / gqs::kQRows), (unsigned)heads, (unsigned)batch),
                           gqs::kThreads, gqs::kSmemBytes, stream>>>(
        static_cast<const float *>(q_rot), static_cast<const float *>(k_cache), static_cast<const float *>(v_cache),
        static_cast<float *>(o), heads, kv_heads, seq, start, cap, scale);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        *err = std::string("gqa prefill f32 attention launch: ") + cudaGetErrorString(e);
        return LA_ERR_CUDA;
    }
    err->clear();
    return LA_OK;
}

}  // namespace la
