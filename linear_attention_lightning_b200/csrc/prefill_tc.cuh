// Blockwise Lightning Attention prefill on the sm_100a tensor cores
// (tcgen05 MMA with TMEM accumulators, operands staged by TMA).
//
// The method ("MINIMAX SIGNAL LAB · M1", §03 Lightning Attention), per block t
// of B = 128 * NSUB tokens of one (batch, head) with slope s:
//   O_t = [(Q_t K_t^T) ⊙ D] V_t + (Q_t ⊙ d_q) S_{t-1}
//   S_t = e^{-s m} S_{t-1} + (K_t ⊙ d_k)^T V_t
// D_ij = e^{-s(i-j)} 1[i>=j], d_q[i] = e^{-s(i+1)}, d_k[j] = e^{-s(m-1-j)}.
//
// Work split. Output columns are independent (o[:, c] needs only v[:, c] and
// S[:, c]), so each CTA owns one (batch, head) and one half of the value
// columns: 2 CTAs per head, each carrying S[:, half] (128 x 64 fp32) across
// the whole sequence. The two halves recompute Q K^T; L2 serves the second
// read of Q and K. A block of 256 rows is handled as two 128-row sub-tiles
// a, b: P_aa = Q_a K_a^T, P_ba = Q_b K_a^T, P_bb = Q_b K_b^T (the all-zero
// upper-right tile is skipped).
//
// Precision. Q K^T runs on the bf16 inputs. Every operand the kernel itself
// produces — P ⊙ D, Q ⊙ d_q, the carried state S and K ⊙ d_k — is rounded to
// fp16 (11 significant bits) rather than bf16 (8): these values are bounded
// (|D|, d_q, d_k <= 1) and an fp16 operand carries an 8x smaller rounding
// error. V is converted bf16 -> fp16 exactly. All accumulation is fp32 and
// the state is carried in fp32.
//
// Per block:
//   QK    (SS MMA bf16, M128 N128 K128)  P tiles -> TMEM (fp32)
//   conv  (warps 4-11, one tile each)    P ⊙ D -> fp16 back into TMEM, and
//                                        Qd = Q ⊙ d_q (fp16) next to it
//   PV    (TS MMA f16, M128 N64)         O  = P V          (A = P from TMEM)
//   dS    (SS MMA f16, M128 N64 K256)    dS = (K ⊙ d_k)^T V
//   QS    (TS MMA f16, M128 N64)         O += Qd S_{t-1}   (B = fp16 S in smem)
//   K ⊙ d_k: the P_ba warpgroup converts K to fp16 K ⊙ d_k in place.
//   warpgroup 3: converts V to fp16 in place, carries
//                S = e^{-s m} S + dS in fp32 registers (fp16 copy -> smem),
//                and writes O (TMEM -> bf16 -> global).
// Warp roles: warp 0 issues TMA, warp 1 issues MMAs, warp 2 owns TMEM,
// warps 4-7 and 8-11 convert P tiles (P_aa and P_bb / P_ba, then K ⊙ d_k),
// warps 12-15 are warpgroup 3. All hand-offs are mbarriers; every wait is bounded.
//
// Shared memory (1024-aligned, 128B-swizzled tiles as TMA writes them):
//   5 x 32 KB Q/K sub-tiles (128 rows x 128 dims), 3 x 16 KB V sub-tiles
//   (128 rows x 64 value columns), 16 KB fp16 state operand, barriers.
// TMEM (512 columns x 128 lanes of 32 bit):
//   [0,128) P_aa | Qd_a   [128,256) P_ba | Qd_b   [256,384) P_bb | dS
//   [384,448) O_a   [448,512) O_b
//
// Range guard (range_guard.cuh). The plain kernel is pass 1: its conversion
// warps also take the largest |q|, |k| (both CTAs of a head convert all of Q and
// K) and warpgroup 3 the largest |v| element (this CTA's value half) and
// |state_in| element of its half; at its end warpgroup 3 writes them as this
// CTA's part of the head's record. Pass 2, launched as its programmatic dependent, decides
// per head and recomputes the flagged heads with power-of-two operand scales.
// With the state carried in place the two CTAs of a head run as a cluster of
// two, exchange their parts, and pass 1 withholds a flagged head's final state.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <string>

#include "../../include/lightning.h"
#include "common.cuh"
#include "range_guard.cuh"
#include "tc_ptx.cuh"

namespace la {
namespace tc {

constexpr int kThreads = 512;
constexpr int kDim = 128;
constexpr int kRows = 128;
constexpr int kQKSlots = 5;
constexpr int kVSlots = 3;
constexpr uint32_t kBoxBytes = 16384;                    // 128 rows x 64 16-bit (128 B rows)
constexpr uint32_t kQKSlotBytes = 2 * kBoxBytes;
constexpr uint32_t kVSlotBytes = kBoxBytes;
constexpr uint32_t kOffQK = 0;
constexpr uint32_t kOffV = kOffQK + kQKSlots * kQKSlotBytes;
constexpr uint32_t kOffS = kOffV + kVSlots * kVSlotBytes;
constexpr uint32_t kOffBar = kOffS + kBoxBytes;
constexpr int kNumBars = 38;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;   // + slack to align the base to 1024
static_assert(kSmemBytes <= 232448, "fits the 227 KB of opt-in shared memory");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColP0 = 0, kColP1 = 128, kColP2 = 256;
constexpr uint32_t kColDS = 320, kColO0 = 384, kColO1 = 448;

__device__ __forceinline__ uint32_t p_col(int tile) { return tile == 0 ? kColP0 : (tile == 1 ? kColP1 : kColP2); }

// barrier indices
constexpr int FULL_QK = 0, EMPTY_QK = 5, FULL_V = 10, EMPTY_V = 13, P_FULL = 16, P_CONV = 19,
              P_FREE = 22, O_FULL = 25, O_FREE = 27, V_CONV = 29, KD_READY = 31, DS_FULL = 32,
              DS_FREE = 33, S_READY = 34, DRAIN = 35,
              // range guard (pass 1 only): SCAN_FIN: the two conversion warpgroups put
              // their maxima in shared memory; PEER: the other CTA's part landed here
              // (state carried in place)
              SCAN_FIN = 36, PEER = 37;
// shared-memory words after the barriers
constexpr uint32_t kMiscTmem = 0, kMiscAbort = 4, kMiscMq = 8, kMiscMk = 12, kMiscMv = 16, kMiscSin = 20,
                   kMiscPeer = 24 /* 4 floats */, kMiscFlag = 40;
static_assert(kMiscFlag + 4 <= 64, "misc words fit their 64 bytes");

// named barriers: 1 / 3 = the two conversion warpgroups, 2 = warpgroup 3
constexpr int kBarConv = 1, kBarWG3 = 2, kBarConv2 = 3;

// Instruction descriptor, kind::f16, fp32 accumulate, M x N; fmt 0 = f16, 1 = bf16.
__host__ __device__ constexpr uint32_t idesc(int M, int N, uint32_t fmt, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescQK = idesc(128, 128, 1, false, false);  // Q x K^T, bf16, both K-major
constexpr uint32_t kIdescPV = idesc(128, 64, 0, false, true);    // P/Qd (TMEM) x V/S (MN-major), f16
constexpr uint32_t kIdescDS = idesc(128, 64, 0, true, true);     // Kd^T (MN-major) x V (MN-major), f16

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Rotation of the five Q/K sub-tile slots between blocks. Slots are reused in
// the order they are released: Q slots free early (after their P tiles are
// converted), K slots only after the block's state MMA.
template <int NSUB>
struct SlotMap {
    int k0, q0, k1, q1, f, t;
    __device__ __forceinline__ void init() {
        t = 0;
        k0 = 0; q0 = 1; k1 = 2; q1 = 3; f = 4;
    }
    __device__ __forceinline__ void advance() {
        ++t;
        if (NSUB == 2) {
            const int nk0 = f, nq0 = q0, nq1 = q1, nk1 = k0, nf = k1;
            k0 = nk0; q0 = nq0; q1 = nq1; k1 = nk1; f = nf;
        } else {
            k0 = (2 * t) % kQKSlots;
            q0 = (2 * t + 1) % kQKSlots;
        }
    }
    __device__ __forceinline__ uint32_t used_mask() const {
        return NSUB == 2 ? ((1u << k0) | (1u << q0) | (1u << k1) | (1u << q1)) : ((1u << k0) | (1u << q0));
    }
};

struct Ctx {
    uint8_t *smem;
    uint32_t sbase;       // shared address of smem
    uint64_t *bars;
    volatile int *abort;
    uint32_t tmem;
};

__device__ __forceinline__ bool wait_bar(const Ctx &c, int idx, uint32_t parity) {
    return ptx::mbar_wait(&c.bars[idx], parity, c.abort);
}

// Group-wide wait: the group's first thread polls the mbarrier, the named
// barrier hands its verdict to every thread of the group, so all of them take
// the same path (none is left behind at a later named barrier).
__device__ __forceinline__ bool group_wait(const Ctx &c, int idx, uint32_t parity, bool leader, int bar_id,
                                           int threads) {
    const bool ok = leader ? wait_bar(c, idx, parity) : true;
    return ptx::named_bar_and(bar_id, threads, ok);
}

// bf16x2 word -> f16x2 word of the values times `scale`
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float scale) {
    const float2 r = ptx::mul2(make_float2(ptx::bf16_lo(w), ptx::bf16_hi(w)), make_float2(scale, scale));
    return ptx::pack_f16(r.x, r.y);
}

// kScaled = false: the plain kernel (pass 1 of the range guard), which also
// measures every (batch, head) into rec[bh].part[half].
// kScaled = true: pass 2, which returns at once for a head whose parts pass the
// guard and otherwise recomputes it with power-of-two operand scales.
template <int NSUB, bool kScaled>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ slopes, int heads,
                  int seq, const float *state_in, __nv_bfloat16 *o, float *state_out, Snapshots sn,
                  rg::RangeRec *rec, const __nv_bfloat16 *qg, const __nv_bfloat16 *kg) {
    constexpr int B = kRows * NSUB;
    constexpr int kLastTile = 2 * NSUB - 2;  // index of the block's last P tile
    extern __shared__ uint8_t smem_raw[];
    // pass 1: pass 2 may be scheduled now (it waits for this grid's completion before
    // reading anything), so that its launch overlaps this one
    if (!kScaled && threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;");
    const uint32_t raw_addr = ptx::smem_addr(smem_raw);
    const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
    Ctx c;
    c.smem = smem_raw + pad;
    c.sbase = raw_addr + pad;
    c.bars = reinterpret_cast<uint64_t *>(c.smem + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c.smem + kOffMisc + kMiscTmem);
    c.abort = reinterpret_cast<volatile int *>(c.smem + kOffMisc + kMiscAbort);
    uint32_t *misc = reinterpret_cast<uint32_t *>(c.smem + kOffMisc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x >> 1, half = blockIdx.x & 1;
    const float s = slopes[bh % heads];
    const float sl2 = s * kLog2e;  // e^{-s n} = 2^{-sl2 n}
    // state carried in place: pass 1 runs the head's two CTAs as a cluster of two
    // (rank = half) and they exchange their parts of the record
    const bool in_place = state_out != nullptr && state_out == state_in;
    // operand scales: q, k, v, P = q k, the carried state, its inverse, and o's inverse
    float f_q = 1.f, f_k = 1.f, f_v = 1.f, f_p = 1.f, f_s = 1.f, f_su = 1.f, f_o = 1.f;
    if constexpr (kScaled) {
        // wait until pass 1 has completed and its records are visible
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const rg::RangePart r = rg::combine(rec[bh].part[0], rec[bh].part[1]);
        const bool flag = !rg::plain_ok(r, s, seq);
        if (threadIdx.x == 0 && half == 0) rec[bh].flag = flag ? 1 : 0;
        if (!flag) return;  // the whole CTA leaves before any set-up
        // the head's largest row norms of q and k (fp32 sums over every row; the
        // state operand's tile, first written after the set-up, holds the reduction)
        float *red = reinterpret_cast<float *>(c.smem + kOffS);
        const size_t hb = (size_t)bh * seq * kDim;
        const float nq = sqrtf(rg::head_max_row_sumsq(qg + hb, seq, 0, 1, red));
        const float nk = sqrtf(rg::head_max_row_sumsq(kg + hb, seq, 0, 1, red));
        const rg::Exps e = rg::scale_exponents(nq, nk, r.mv, r.msin, s, seq);
        f_q = rg::pow2(e.a);
        f_k = rg::pow2(e.b);
        f_v = rg::pow2(e.c);
        f_p = rg::pow2(e.a + e.b);
        f_s = rg::pow2(e.b + e.c);
        f_su = rg::pow2(-(e.b + e.c));
        f_o = rg::pow2(-(e.a + e.b + e.c));
    }
    const int nblk = (seq + B - 1) / B;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) ptx::mbar_init(&c.bars[i], 1);
        ptx::mbar_init(&c.bars[SCAN_FIN], 2);  // both conversion warpgroups
        *c.abort = 0;
        misc[kMiscMq / 4] = 0u;
        misc[kMiscMk / 4] = 0u;
        misc[kMiscMv / 4] = 0u;
        misc[kMiscSin / 4] = 0u;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
    }
    if (warp == 2) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    // the other CTA's barriers are initialised before either CTA writes into them
    if (!kScaled && in_place) ptx::cluster_sync();
    ptx::tc_fence_after();
    c.tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t qk_par = 0, qk_issued = 0;
            int vtile = 0, vissued = 0;
            SlotMap<NSUB> sm;
            sm.init();
            bool ok = true;
            auto load_qk = [&](int slot, const CUtensorMap *map, int row) -> bool {
                if (!wait_bar(c, EMPTY_QK + slot, ((qk_par >> slot) & 1u) ^ 1u)) return false;
                qk_par ^= 1u << slot;
                qk_issued |= 1u << slot;
                uint8_t *dst = c.smem + kOffQK + slot * kQKSlotBytes;
                ptx::mbar_arrive_expect_tx(&c.bars[FULL_QK + slot], kQKSlotBytes);
                ptx::tma_load_3d(dst, map, &c.bars[FULL_QK + slot], 0, row, bh);
                ptx::tma_load_3d(dst + kBoxBytes, map, &c.bars[FULL_QK + slot], 64, row, bh);
                return true;
            };
            auto load_v = [&](int n, int row) -> bool {
                const int slot = n % kVSlots;
                if (!wait_bar(c, EMPTY_V + slot, ((uint32_t)(n / kVSlots) & 1u) ^ 1u)) return false;
                ptx::mbar_arrive_expect_tx(&c.bars[FULL_V + slot], kVSlotBytes);
                ptx::tma_load_3d(c.smem + kOffV + slot * kVSlotBytes, &tm_v, &c.bars[FULL_V + slot],
                                 64 * half, row, bh);
                vissued = n + 1;
                return true;
            };
            for (int t = 0; t < nblk && ok; ++t) {
                const int row0 = t * B;
                ok = ok && load_qk(sm.k0, &tm_k, row0);
                ok = ok && load_qk(sm.q0, &tm_q, row0);
                ok = ok && load_v(vtile, row0);
                if (NSUB == 2) {
                    ok = ok && load_qk(sm.q1, &tm_q, row0 + kRows);
                    ok = ok && load_qk(sm.k1, &tm_k, row0 + kRows);
                    ok = ok && load_v(vtile + 1, row0 + kRows);
                }
                vtile += NSUB;
                sm.advance();
            }
            // every copy issued lands before the CTA exits (already true unless
            // some role gave up early)
            volatile int never = 0;
            for (int sl = 0; sl < kQKSlots; ++sl)
                if (qk_issued & (1u << sl))
                    ptx::mbar_wait(&c.bars[FULL_QK + sl], ((qk_par >> sl) & 1u) ^ 1u, &never);
            for (int n = vissued > kVSlots ? vissued - kVSlots : 0; n < vissued; ++n)
                ptx::mbar_wait(&c.bars[FULL_V + n % kVSlots], (uint32_t)(n / kVSlots) & 1u, &never);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t qk_par = 0;
            int vtile = 0;
            SlotMap<NSUB> sm;
            sm.init();
            const uint32_t tm = c.tmem;
            // Descriptors are built once; per MMA only the start-address field
            // moves (a plain add on the low bits: shared addresses stay < 2^18).
            const uint64_t qk_kmaj = sdesc(c.sbase + kOffQK, 16u, 1024u);
            const uint64_t qk_mnmaj = sdesc(c.sbase + kOffQK, kBoxBytes, 1024u);
            const uint64_t v_mnmaj = sdesc(c.sbase + kOffV, kBoxBytes, 1024u);
            const uint64_t s_mnmaj = sdesc(c.sbase + kOffS, kBoxBytes, 1024u);
            auto qk_off = [](int slot) { return (uint64_t)((uint32_t)slot * (kQKSlotBytes >> 4)); };
            auto v_off = [](int n) { return (uint64_t)((uint32_t)(n % kVSlots) * (kVSlotBytes >> 4)); };
            auto wait_qk = [&](int slot) -> bool {
                const bool r = wait_bar(c, FULL_QK + slot, (qk_par >> slot) & 1u);
                qk_par ^= 1u << slot;
                return r;
            };
            auto issue_qk = [&](uint32_t dcol, int qslot, int kslot) {
                const uint64_t a0 = qk_kmaj + qk_off(qslot), b0 = qk_kmaj + qk_off(kslot);
                const uint32_t d = tm + dcol;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t koff = (uint64_t)(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4);
                    ptx::mma_ss(d, a0 + koff, b0 + koff, kIdescQK, k > 0);
                }
            };
            auto issue_ts = [&](uint32_t dcol, uint32_t acol, uint64_t b0, bool acc) {
                const uint32_t d = tm + dcol, a = tm + acol;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    ptx::mma_ts(d, a + 8u * k, b0 + (uint64_t)(k * (2048 >> 4)), kIdescPV, acc || k > 0);
            };
            auto issue_ds = [&](int kslot, int vn, bool acc) {
                const uint64_t a0 = qk_mnmaj + qk_off(kslot), b0 = v_mnmaj + v_off(vn);
                const uint32_t d = tm + kColDS;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    ptx::mma_ss(d, a0 + (uint64_t)(k * (2048 >> 4)), b0 + (uint64_t)(k * (2048 >> 4)), kIdescDS,
                                acc || k > 0);
            };
            bool ok = true;
            for (int t = 0; t < nblk && ok; ++t) {
                const uint32_t par = t & 1, fpar = par ^ 1u;
                const int va = vtile, vb = vtile + 1;
                // P_aa = Q_a K_a^T
                ok = wait_qk(sm.k0) && wait_qk(sm.q0) && wait_bar(c, P_FREE + 0, fpar);
                if (!ok) break;
                ptx::tc_fence_after();
                issue_qk(kColP0, sm.q0, sm.k0);
                ptx::mma_commit(&c.bars[P_FULL + 0]);
                if (NSUB == 2) {
                    // P_ba = Q_b K_a^T
                    ok = wait_qk(sm.q1) && wait_bar(c, P_FREE + 1, fpar);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    issue_qk(kColP1, sm.q1, sm.k0);
                    ptx::mma_commit(&c.bars[P_FULL + 1]);
                    // P_bb = Q_b K_b^T; its upper half is the dS region of the previous block
                    ok = wait_qk(sm.k1) && wait_bar(c, P_FREE + 2, fpar) && wait_bar(c, DS_FREE, fpar);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    issue_qk(kColP2, sm.q1, sm.k1);
                    ptx::mma_commit(&c.bars[P_FULL + 2]);
                }
                // O_a = P_aa V_a
                ok = wait_bar(c, V_CONV + 0, par) && wait_bar(c, P_CONV + 0, par) && wait_bar(c, O_FREE + 0, fpar);
                if (!ok) break;
                ptx::tc_fence_after();
                issue_ts(kColO0, kColP0, v_mnmaj + v_off(va), false);
                if (NSUB == 2) {
                    // O_b = P_ba V_a + P_bb V_b
                    ok = wait_bar(c, P_CONV + 1, par) && wait_bar(c, O_FREE + 1, fpar);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    issue_ts(kColO1, kColP1, v_mnmaj + v_off(va), false);
                    ok = wait_bar(c, V_CONV + 1, par) && wait_bar(c, P_CONV + 2, par);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    issue_ts(kColO1, kColP2, v_mnmaj + v_off(vb), true);
                    ptx::mma_commit(&c.bars[P_FREE + 2]);
                }
                // dS = (K ⊙ d_k)^T V (for B = 128 the previous dS must have been read first)
                ok = wait_bar(c, KD_READY, par) && (NSUB == 2 || wait_bar(c, DS_FREE, fpar));
                if (!ok) break;
                ptx::tc_fence_after();
                issue_ds(sm.k0, va, false);
                if (NSUB == 2) issue_ds(sm.k1, vb, true);
                // O += Qd S_{t-1}
                ok = wait_bar(c, S_READY, par);
                if (!ok) break;
                ptx::tc_fence_after();
                issue_ts(kColO0, kColP0 + 64, s_mnmaj, true);
                if (NSUB == 2) issue_ts(kColO1, kColP1 + 64, s_mnmaj, true);
                ptx::mma_commit(&c.bars[P_FREE + 0]);
                ptx::mma_commit(&c.bars[O_FULL + 0]);
                if (NSUB == 2) {
                    ptx::mma_commit(&c.bars[P_FREE + 1]);
                    ptx::mma_commit(&c.bars[O_FULL + 1]);
                }
                // dS is ready and S_{t-1} is no longer read: the state may move on
                ptx::mma_commit(&c.bars[DS_FULL]);
                ptx::mma_commit(&c.bars[EMPTY_QK + sm.k0]);
                ptx::mma_commit(&c.bars[EMPTY_V + va % kVSlots]);
                if (NSUB == 2) {
                    ptx::mma_commit(&c.bars[EMPTY_QK + sm.k1]);
                    ptx::mma_commit(&c.bars[EMPTY_V + vb % kVSlots]);
                }
                vtile += NSUB;
                sm.advance();
            }
            // drain: every MMA issued has completed before TMEM is released
            ptx::mma_commit(&c.bars[DRAIN]);
            volatile int never = 0;
            ptx::mbar_wait(&c.bars[DRAIN], 0, &never);
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------------------ P conversion
        // Two warpgroups, each converting whole P tiles: group 0 takes P_aa (and
        // P_bb), group 1 takes P_ba. Thread r owns TMEM lane r = row r of the tile.
        const int grp = (warp - 4) >> 2;
        const int r = threadIdx.x - 128 - 128 * grp;
        const bool leader = r == 0;
        const int bar_id = grp == 0 ? kBarConv : kBarConv2;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        // tab[u] = e^{-s(15-u)}: decay inside a group of 16 keys, relative to its last key
        const float step = ptx::ex2(-sl2);  // e^{-s}
        float tab[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) tab[u] = ptx::ex2(-sl2 * (float)(15 - u)) * f_p;
        uint32_t mxq = 0u, mxk = 0u;  // pass 1: packed maxima of |q| and |k| this thread converted
        uint32_t qk_par = 0;
        SlotMap<NSUB> sm;
        sm.init();
        for (int t = 0; t < nblk; ++t) {
            const uint32_t par = t & 1;
            for (int tile = grp; tile <= kLastTile; tile += 2) {
                // tile 0: P_aa (rows a, keys a, Qd_a); 1: P_ba (rows b, keys a, Qd_b); 2: P_bb
                const uint32_t col = p_col(tile);
                const int i = (tile == 0 ? 0 : kRows) + r;
                const int j0 = tile == 2 ? kRows : 0;
                if (!group_wait(c, P_FULL + tile, par, leader, bar_id, 128)) goto conv_done;
                ptx::tc_fence_after();
#pragma unroll 1
                for (int pass = 0; pass < 2; ++pass) {
                    // fp32 columns [64 pass, 64 pass + 64) -> fp16 pairs in [32 pass, 32 pass + 32);
                    // the destination was read by this same thread in an earlier pass
                    uint32_t va[32], vb[32];
                    ptx::tmem_ld32(c.tmem + lane_off + col + 64 * pass, va);
                    ptx::tmem_ld32(c.tmem + lane_off + col + 64 * pass + 32, vb);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        uint32_t out[16];
#pragma unroll
                        for (int g = 0; g < 2; ++g) {
                            const uint32_t *v = (hb == 0 ? va : vb) + 16 * g;
                            const int jb = j0 + 64 * pass + 32 * hb + 16 * g;
                            const int dlast = i - (jb + 15);
                            float p[16];
                            if (dlast >= 0) {
                                const float wb = ptx::ex2(-sl2 * (float)dlast);
#pragma unroll
                                for (int u = 0; u < 16; u += 2) {
                                    const float2 t2 = ptx::mul2(make_float2(__uint_as_float(v[u]), __uint_as_float(v[u + 1])),
                                                                make_float2(tab[u], tab[u + 1]));
                                    const float2 r2 = ptx::mul2(t2, make_float2(wb, wb));
                                    p[u] = r2.x;
                                    p[u + 1] = r2.y;
                                }
                            } else if (i < jb) {
                                // every key of the group is after row i: masked
#pragma unroll
                                for (int u = 0; u < 16; ++u) p[u] = 0.f;
                            } else {
                                // the group holds the diagonal key jb + d0: walk down from it
                                const int d0 = i - jb;
                                float w = f_p;
#pragma unroll
                                for (int u = 15; u >= 0; --u) {
                                    const bool live = u <= d0;
                                    p[u] = live ? __uint_as_float(v[u]) * w : 0.f;
                                    w = live ? w * step : w;
                                }
                            }
#pragma unroll
                            for (int u = 0; u < 8; ++u) out[8 * g + u] = ptx::pack_f16(p[2 * u], p[2 * u + 1]);
                        }
                        __syncwarp();
                        ptx::tmem_st16(c.tmem + lane_off + col + 32 * pass + 16 * hb, out);
                    }
                }
                if (tile < 2) {
                    // Qd = Q ⊙ d_q for this row, from the swizzled Q sub-tile, into columns [64, 128)
                    const int qslot = tile == 0 ? sm.q0 : sm.q1;
                    if (!group_wait(c, FULL_QK + qslot, (qk_par >> qslot) & 1u, leader, bar_id, 128))
                        goto conv_done;
                    const float dq = ptx::ex2(-sl2 * (float)(i + 1)) * f_q;
                    const uint8_t *qrow = c.smem + kOffQK + qslot * kQKSlotBytes + r * 128;
#pragma unroll
                    for (int hb = 0; hb < 4; ++hb) {
                        uint32_t out[16];
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            const int chunk = 4 * (hb & 1) + cc;
                            const uint4 q4 = *reinterpret_cast<const uint4 *>(
                                qrow + (hb >> 1) * kBoxBytes + ((chunk ^ (r & 7)) << 4));
                            if (!kScaled)
                                mxq = rg::maxabs_bf16x2(mxq, rg::maxabs_bf16x2(rg::maxabs_bf16x2(q4.x, q4.y),
                                                                               rg::maxabs_bf16x2(q4.z, q4.w)));
                            out[4 * cc + 0] = bf16x2_to_f16x2(q4.x, dq);
                            out[4 * cc + 1] = bf16x2_to_f16x2(q4.y, dq);
                            out[4 * cc + 2] = bf16x2_to_f16x2(q4.z, dq);
                            out[4 * cc + 3] = bf16x2_to_f16x2(q4.w, dq);
                        }
                        __syncwarp();
                        ptx::tmem_st16(c.tmem + lane_off + col + 64 + 16 * hb, out);
                    }
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                ptx::named_bar_sync(bar_id, 128);
                if (leader) ptx::mbar_arrive(&c.bars[P_CONV + tile]);
                if (tile == 0 && leader) ptx::mbar_arrive(&c.bars[EMPTY_QK + sm.q0]);  // Q_a done
                if (tile == 2) {
                    // Q_b is done once P_bb's Q K^T has run (it has: P_bb was full) and
                    // the other group has built Qd_b
                    if (!group_wait(c, P_CONV + 1, par, leader, bar_id, 128)) goto conv_done;
                    if (leader) ptx::mbar_arrive(&c.bars[EMPTY_QK + sm.q1]);
                }
            }
            if (grp == NSUB - 1) {
                // K sub-tiles: bf16 -> fp16 K ⊙ d_k in place, once the block's Q K^T is done
                const int m = min(B, seq - t * B);
                if (!group_wait(c, P_FULL + kLastTile, par, leader, bar_id, 128)) goto conv_done;
                for (int sub = 0; sub < NSUB; ++sub) {
                    const int kslot = sub == 0 ? sm.k0 : sm.k1;
                    // full-barrier wait: makes the TMA bytes visible to these threads
                    if (!group_wait(c, FULL_QK + kslot, (qk_par >> kslot) & 1u, leader, bar_id, 128)) goto conv_done;
                    const int j = sub * kRows + r;
                    const float dk = j < m ? ptx::ex2(-sl2 * (float)(m - 1 - j)) * f_k : 0.f;
                    uint8_t *krow = c.smem + kOffQK + kslot * kQKSlotBytes + r * 128;
                    uint4 x[16];
#pragma unroll
                    for (int ch = 0; ch < 16; ++ch)
                        x[ch] = *reinterpret_cast<const uint4 *>(krow + (ch >> 3) * kBoxBytes + (((ch & 7) ^ (r & 7)) << 4));
                    if (!kScaled) {
#pragma unroll
                        for (int ch = 0; ch < 16; ++ch)
                            mxk = rg::maxabs_bf16x2(mxk, rg::maxabs_bf16x2(rg::maxabs_bf16x2(x[ch].x, x[ch].y),
                                                                           rg::maxabs_bf16x2(x[ch].z, x[ch].w)));
                    }
#pragma unroll
                    for (int ch = 0; ch < 16; ++ch) {
                        uint4 y;
                        y.x = bf16x2_to_f16x2(x[ch].x, dk); y.y = bf16x2_to_f16x2(x[ch].y, dk);
                        y.z = bf16x2_to_f16x2(x[ch].z, dk); y.w = bf16x2_to_f16x2(x[ch].w, dk);
                        *reinterpret_cast<uint4 *>(krow + (ch >> 3) * kBoxBytes + (((ch & 7) ^ (r & 7)) << 4)) = y;
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::named_bar_sync(bar_id, 128);
                if (leader) ptx::mbar_arrive(&c.bars[KD_READY]);
            }
            qk_par ^= sm.used_mask();
            sm.advance();
        }
    conv_done:
        if (!kScaled) {
            // the group's maxima into shared memory for the record (rows past seq read
            // as zeros and change no maximum)
            const auto as_float = [](uint32_t w) { return fmaxf(fabsf(rg::bf_lo(w)), fabsf(rg::bf_hi(w))); };
            const float mq = rg::warp_max_nonneg(as_float(mxq)), mk = rg::warp_max_nonneg(as_float(mxk));
            if (lane == 0) {
                atomicMax(misc + kMiscMq / 4, __float_as_uint(mq));
                atomicMax(misc + kMiscMk / 4, __float_as_uint(mk));
            }
            ptx::named_bar_sync(bar_id, 128);
            if (leader) ptx::mbar_arrive(&c.bars[SCAN_FIN]);
        }
    } else if (warp >= 12) {
        // ------------------------------------------------------------ warpgroup 3
        const int r = threadIdx.x - 384;  // row of V / K sub-tiles, key-dim row of S, output row
        const bool leader = r == 0;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        float S[64];
        const size_t sbase = (size_t)bh * kDim * kDim + (size_t)r * kDim + 64 * half;
        float msin = 0.f;     // pass 1: the largest |state_in| element of this thread
        uint32_t mxv = 0u;    // pass 1: packed maximum of |v| this thread converted
        if (state_in) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float4 x = *reinterpret_cast<const float4 *>(state_in + sbase + 4 * q);
                if (!kScaled) msin = fmaxf(msin, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
                S[4 * q] = x.x * f_s; S[4 * q + 1] = x.y * f_s; S[4 * q + 2] = x.z * f_s; S[4 * q + 3] = x.w * f_s;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 64; ++q) S[q] = 0.f;
        }
        uint8_t *srow = c.smem + kOffS + r * 128;
        auto write_state_operand = [&]() {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 wv;
                wv.x = ptx::pack_f16(S[8 * ch + 0], S[8 * ch + 1]);
                wv.y = ptx::pack_f16(S[8 * ch + 2], S[8 * ch + 3]);
                wv.z = ptx::pack_f16(S[8 * ch + 4], S[8 * ch + 5]);
                wv.w = ptx::pack_f16(S[8 * ch + 6], S[8 * ch + 7]);
                *reinterpret_cast<uint4 *>(srow + ((ch ^ (r & 7)) << 4)) = wv;
            }
            ptx::fence_proxy_async_smem();
            ptx::named_bar_sync(kBarWG3, 128);
            if (leader) ptx::mbar_arrive(&c.bars[S_READY]);
        };
        write_state_operand();
        uint32_t qk_par = 0;
        SlotMap<NSUB> sm;
        sm.init();
        int vtile = 0;
        for (int t = 0; t < nblk; ++t) {
            const uint32_t par = t & 1;
            const int m = min(B, seq - t * B);
            // V sub-tiles: bf16 -> fp16 in place
            for (int sub = 0; sub < NSUB; ++sub) {
                const int n = vtile + sub;
                if (!group_wait(c, FULL_V + n % kVSlots, (uint32_t)(n / kVSlots) & 1u, leader, kBarWG3, 128))
                    goto wg3_done;
                uint8_t *vrow = c.smem + kOffV + (n % kVSlots) * kVSlotBytes + r * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    // walk the row in its swizzled chunk order: the 32 rows of a warp
                    // then hit 8 different bank groups instead of one
                    uint4 *pv = reinterpret_cast<uint4 *>(vrow + ((ch ^ (r & 7)) << 4));
                    uint4 x = *pv;
                    if (!kScaled)
                        mxv = rg::maxabs_bf16x2(mxv, rg::maxabs_bf16x2(rg::maxabs_bf16x2(x.x, x.y),
                                                                       rg::maxabs_bf16x2(x.z, x.w)));
                    x.x = bf16x2_to_f16x2(x.x, f_v); x.y = bf16x2_to_f16x2(x.y, f_v);
                    x.z = bf16x2_to_f16x2(x.z, f_v); x.w = bf16x2_to_f16x2(x.w, f_v);
                    *pv = x;
                }
                ptx::fence_proxy_async_smem();
                ptx::named_bar_sync(kBarWG3, 128);
                if (leader) ptx::mbar_arrive(&c.bars[V_CONV + sub]);
            }
            // state: S_t = e^{-s m} S_{t-1} + dS
            if (!group_wait(c, DS_FULL, par, leader, kBarWG3, 128)) goto wg3_done;
            ptx::tc_fence_after();
            {
                const float dblock = ptx::ex2(-sl2 * (float)m);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t d[32];
                    ptx::tmem_ld32(c.tmem + lane_off + kColDS + 32 * hh, d);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 32; ++q) S[32 * hh + q] = fmaf(dblock, S[32 * hh + q], __uint_as_float(d[q]));
                }
            }
            ptx::tc_fence_before();
            ptx::named_bar_sync(kBarWG3, 128);
            if (leader) ptx::mbar_arrive(&c.bars[DS_FREE]);
            write_state_operand();
            // prefix-cache snapshot of S_t (this thread's key-dim row, its value half)
            if (float *snap = snapshot_at(sn, bh, t * B + m, kDim)) {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    *reinterpret_cast<float4 *>(snap + (size_t)r * kDim + 64 * half + 4 * q) =
                        make_float4(S[4 * q] * f_su, S[4 * q + 1] * f_su, S[4 * q + 2] * f_su, S[4 * q + 3] * f_su);
            }

            // outputs of this block: O (TMEM, fp32) -> bf16 -> global, 32 columns at a time
            for (int sub = 0; sub < NSUB; ++sub) {
                if (!group_wait(c, O_FULL + sub, par, leader, kBarWG3, 128)) goto wg3_done;
                ptx::tc_fence_after();
                const uint32_t col = sub == 0 ? kColO0 : kColO1;
                const int row = t * B + sub * kRows + r;
                uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)bh * seq + row) * kDim + 64 * half);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t a[32];
                    ptx::tmem_ld32(c.tmem + lane_off + col + 32 * hh, a);
                    ptx::tmem_ld_wait();
                    if (hh == 1) {
                        ptx::tc_fence_before();
                        ptx::named_bar_sync(kBarWG3, 128);
                        if (leader) ptx::mbar_arrive(&c.bars[O_FREE + sub]);
                    }
                    if (row < seq) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[4 * hh + q] = make_uint4(
                                ptx::pack_bf16(__uint_as_float(a[8 * q + 0]) * f_o, __uint_as_float(a[8 * q + 1]) * f_o),
                                ptx::pack_bf16(__uint_as_float(a[8 * q + 2]) * f_o, __uint_as_float(a[8 * q + 3]) * f_o),
                                ptx::pack_bf16(__uint_as_float(a[8 * q + 4]) * f_o, __uint_as_float(a[8 * q + 5]) * f_o),
                                ptx::pack_bf16(__uint_as_float(a[8 * q + 6]) * f_o, __uint_as_float(a[8 * q + 7]) * f_o));
                    }
                }
            }
            qk_par ^= sm.used_mask();
            sm.advance();
            vtile += NSUB;
        }
        {
            bool write_state = state_out != nullptr;
            if (!kScaled) {
                // range guard, pass 1: this warpgroup's maxima join the conversion
                // warpgroups' in shared memory, and the leader writes the CTA's part of
                // the head's record once those have arrived (they finished converting
                // before this block's outputs were ready, so the wait is short)
                const float mv = rg::warp_max_nonneg(fmaxf(fabsf(rg::bf_lo(mxv)), fabsf(rg::bf_hi(mxv))));
                const float ms = rg::warp_max_nonneg(msin);
                if (lane == 0) {
                    atomicMax(misc + kMiscMv / 4, __float_as_uint(mv));
                    atomicMax(misc + kMiscSin / 4, __float_as_uint(ms));
                }
                ptx::named_bar_sync(kBarWG3, 128);
                bool ok = true;
                if (leader) {
                    ok = wait_bar(c, SCAN_FIN, 0);
                    if (ok) {
                        const rg::RangePart mine{__uint_as_float(misc[kMiscMq / 4]), __uint_as_float(misc[kMiscMk / 4]),
                                                 __uint_as_float(misc[kMiscMv / 4]), __uint_as_float(misc[kMiscSin / 4])};
                        rec[bh].part[half] = mine;
                        if (in_place) {
                            // with the state carried in place, the two CTAs exchange their parts
                            // and decide here: a flagged head's final state is not written
                            // (pass 2 still reads it as state_in)
                            float *peer = reinterpret_cast<float *>(c.smem + kOffMisc + kMiscPeer);
                            const uint32_t other = (uint32_t)half ^ 1u;
                            const float v4[4] = {mine.mq, mine.mk, mine.mv, mine.msin};
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ptx::map_to_rank(peer + i, other)),
                                             "f"(v4[i])
                                             : "memory");
                            asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                                             ptx::map_to_rank(&c.bars[PEER], other))
                                         : "memory");
                            ok = ptx::mbar_wait_cluster(&c.bars[PEER], 0, c.abort);
                            if (ok) {
                                const rg::RangePart r =
                                    rg::combine(mine, rg::RangePart{peer[0], peer[1], peer[2], peer[3]});
                                misc[kMiscFlag / 4] = rg::plain_ok(r, s, seq) ? 0u : 1u;
                            }
                        }
                    }
                }
                // the leader's result (and the flag, written before this barrier) to the group
                if (!ptx::named_bar_and(kBarWG3, 128, ok)) goto wg3_done;
                if (in_place) write_state = write_state && misc[kMiscFlag / 4] == 0u;
            }
            if (write_state) {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    *reinterpret_cast<float4 *>(state_out + sbase + 4 * q) =
                        make_float4(S[4 * q] * f_su, S[4 * q + 1] * f_su, S[4 * q + 2] * f_su, S[4 * q + 3] * f_su);
            }
        }
    wg3_done:;
    }

    ptx::tc_fence_before();
    __syncthreads();
    // neither CTA of a cluster leaves while the other may still write into its shared memory
    if (!kScaled && in_place) ptx::cluster_sync();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(c.tmem, kTmemCols);
    }
}

}  // namespace tc

// The tensor-core kernel covers bf16 inputs, head dim 128 and blocks of 128 or 256.
inline bool tc_supports(bool bf16, int dim, int block) {
    return bf16 && dim == 128 && (block == 128 || block == 256);
}

namespace tc {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn(std::string *err) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) {
            *err = "cuTensorMapEncodeTiled is not available from the driver";
            return nullptr;
        }
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [batch*heads][seq][128] bf16 viewed as a 3-D tensor; boxes of 64 dims x
// 128 rows, 128-byte swizzle; rows past seq read as zeros and are clipped on
// store.
inline bool make_map(CUtensorMap *map, const void *base, int seq, long long bh, std::string *err) {
    auto fn = encode_fn(err);
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kDim, (cuuint64_t)seq, (cuuint64_t)bh};
    cuuint64_t strides[2] = {(cuuint64_t)kDim * 2, (cuuint64_t)seq * kDim * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kRows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = "cuTensorMapEncodeTiled failed (CUresult " + std::to_string((int)r) + ")";
        return false;
    }
    return true;
}

}  // namespace tc

// Workspace of one single-CTA prefill: the range guard's record per (batch, head), 48 bytes.
inline size_t tc_workspace_bytes(long long batch_heads) { return (size_t)batch_heads * sizeof(rg::RangeRec); }

// Two launches on `stream`: the plain kernel, which measures every (batch, head)
// into rec (tc_workspace_bytes of the caller's workspace), then pass 2, its
// programmatic dependent, which recomputes the heads the guard flags.
inline la_status launch_tc(const void *q, const void *k, const void *v, const float *slopes, int batch,
                           int heads, int seq, int block, const float *state_in, void *o, float *state_out,
                           Snapshots sn, rg::RangeRec *rec, cudaStream_t stream, std::string *err) {
    const long long bh = (long long)batch * heads;
    if (!rec) {
        *err = "the single-CTA prefill needs its workspace (the range guard's records)";
        return LA_ERR_INVALID_ARG;
    }
    CUtensorMap mq, mk, mv;
    if (!tc::make_map(&mq, q, seq, bh, err) || !tc::make_map(&mk, k, seq, bh, err) ||
        !tc::make_map(&mv, v, seq, bh, err))
        return LA_ERR_CUDA;
    using Kernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, const float *, int, int, const float *,
                            __nv_bfloat16 *, float *, Snapshots, rg::RangeRec *, const __nv_bfloat16 *,
                            const __nv_bfloat16 *);
    const Kernel passes[2] = {block == 256 ? tc::prefill_tc_kernel<2, false> : tc::prefill_tc_kernel<1, false>,
                              block == 256 ? tc::prefill_tc_kernel<2, true> : tc::prefill_tc_kernel<1, true>};
    // the state carried in place: pass 1 runs each head's two CTAs as a cluster of two
    const bool in_place = state_out != nullptr && state_out == state_in;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(bh * 2));
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = tc::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute cluster, pdl;
    cluster.id = cudaLaunchAttributeClusterDimension;
    cluster.val.clusterDim.x = 2;
    cluster.val.clusterDim.y = 1;
    cluster.val.clusterDim.z = 1;
    // pass 2 is pass 1's programmatic dependent (it starts with griddepcontrol.wait)
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    for (int pass = 0; pass < 2; ++pass) {
        cfg.attrs = pass == 0 ? &cluster : &pdl;
        cfg.numAttrs = pass == 0 ? (in_place ? 1 : 0) : 1;
        cudaError_t e = cudaFuncSetAttribute(passes[pass], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)tc::kSmemBytes);
        if (e != cudaSuccess) {
            *err = std::string("cudaFuncSetAttribute(prefill_tc): ") + cudaGetErrorString(e);
            return LA_ERR_CUDA;
        }
        e = cudaLaunchKernelEx(&cfg, passes[pass], mq, mk, mv, slopes, heads, seq, state_in,
                               static_cast<__nv_bfloat16 *>(o), state_out, sn, rec, static_cast<const __nv_bfloat16 *>(q),
                               static_cast<const __nv_bfloat16 *>(k));
        if (e != cudaSuccess) {
            *err = std::string("prefill_tc launch: ") + cudaGetErrorString(e);
            return LA_ERR_CUDA;
        }
    }
    err->clear();
    return LA_OK;
}

}  // namespace la
