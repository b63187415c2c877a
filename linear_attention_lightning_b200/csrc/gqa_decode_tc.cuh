// Partial softmax of one decode step of the softmax GQA layer on the tensor
// cores (bf16 cache, head dim 128): the same chunked split as gqa_partial_kernel
// ("MINIMAX SIGNAL LAB · M1", §02 and §04; readings as in gqa_decode.cuh), with
// the scores and the weighted values as tcgen05 MMAs.
//
// One CTA per (chunk of kGqaChunk positions, KV head, sequence). The group's
// query heads (at most 32, one softmax lane each) are the first rows of a 128-row Q tile; the other
// rows are zero, so the MMAs do 16x the useful work, which the step can afford
// (it is bound by reading the cache). Per key tile j of 128 positions:
//   S_j = Q K_j^T      SS MMA bf16, M128 N128 K128 -> TMEM, double-buffered
//                      (S_{j+2} may be computed while tile j's softmax runs)
//   softmax warp:      one lane per head: row max, P = 2^(S log2 e - m) as bf16
//                      over the first 64 columns of S_j; the running max is
//                      raised only past a margin of 2^8 (O rescaled in TMEM)
//   O += P V_j         TS MMA bf16, M128 N128 K128
// At the end the warp writes the chunk's max (natural units), sum of weights
// and unnormalised weighted values in gqa_partial_kernel's format, for
// gqa_combine_kernel. Positions past pos[b] are masked in S; in the chunk's
// last tile the value rows past pos[b] are zeroed in shared memory before
// P V (the cache there may hold anything, and 0 x NaN is NaN). The queries
// come in rotated and scaled (fp32, from gqa_append_kernel) and are rounded
// to bf16 for the MMA.
//
// Warp roles: warp 0 TMA, warp 1 MMA (one elected lane issues), warp 2 TMEM,
// warp 3 builds the Q tile, warp 4 the softmax. Every wait is bounded.
// Shared memory: Q tile 32 KB, 2 stages of K and of V (32 KB each). TMEM:
// [0,128) S_0/P_0, [128,256) S_1/P_1, [256,384) O.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "gqa_decode.cuh"
#include "gqa_prefill.cuh"
#include "tc_ptx.cuh"

namespace la {
namespace gqd {

constexpr int kThreads = 160;
constexpr int kRows = 128;
constexpr uint32_t kBoxBytes = gqp::kBoxBytes;     // 128 rows x 64 bf16
constexpr uint32_t kTileBytes = gqp::kTileBytes;   // 128 rows x 128 dims
constexpr int kStages = 2;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
constexpr int kNumBars = 16;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;

// One P_FULL per S buffer: with S double-buffered the softmax may finish tile j+1 before the
// MMA warp has waited for tile j's weights, so a single barrier could run two phases ahead of
// its waiter; per buffer, the next use of a buffer needs this one consumed.
constexpr int Q_READY = 0, K_FULL = 1 /* 2 */, K_EMPTY = 3 /* 2 */, V_FULL = 5 /* 2 */, V_EMPTY = 7 /* 2 */,
              S_FULL = 9 /* 2 */, P_FULL = 11 /* 2 */, O_READY = 13, O_FINAL = 14, DRAIN = 15;

constexpr float kLn2 = 0.6931471805599453f;

// grid (splits, kv_heads, batch), kThreads. tm_k, tm_v: caches [batch*kv_heads][cap][128].
__global__ void __launch_bounds__(kThreads, 1)
gqd_partial_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const float *__restrict__ q_rot, const int *__restrict__ pos, int heads, int kv_heads, int cap,
                   int splits, float *__restrict__ part_m, float *__restrict__ part_l, float *__restrict__ part_o) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = ptx::smem_addr(smem_raw);
    const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int group = heads / kv_heads, h0 = hk * group;
    const int P = pos[b];
    const bool bad = P < 0 || P >= cap;  // recorded by the append kernel; read nothing then
    const int p0 = split * kGqaChunk, p1 = bad ? p0 : min(p0 + kGqaChunk, P + 1);
    const int nt = p1 > p0 ? (p1 - p0 + kRows - 1) / kRows : 0;
    const int bkv = b * kv_heads + hk;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) ptx::mbar_init(&bars[i], 1);
        *abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
    }
    if (warp == 2) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int st = j & 1;
                const uint32_t epar = ((uint32_t)(j >> 1) & 1u) ^ 1u;
                if (j >= kStages && !ptx::mbar_wait(&bars[K_EMPTY + st], epar, abort)) break;
                uint8_t *kd = smem + kOffK + st * kTileBytes;
                ptx::mbar_arrive_expect_tx(&bars[K_FULL + st], kTileBytes);
                ptx::tma_load_3d(kd, &tm_k, &bars[K_FULL + st], 0, p0 + kRows * j, bkv);
                ptx::tma_load_3d(kd + kBoxBytes, &tm_k, &bars[K_FULL + st], 64, p0 + kRows * j, bkv);
                k_issued = j + 1;
                if (j >= kStages && !ptx::mbar_wait(&bars[V_EMPTY + st], epar, abort)) break;
                uint8_t *vd = smem + kOffV + st * kTileBytes;
                ptx::mbar_arrive_expect_tx(&bars[V_FULL + st], kTileBytes);
                ptx::tma_load_3d(vd, &tm_v, &bars[V_FULL + st], 0, p0 + kRows * j, bkv);
                ptx::tma_load_3d(vd + kBoxBytes, &tm_v, &bars[V_FULL + st], 64, p0 + kRows * j, bkv);
                v_issued = j + 1;
            }
            // let every copy issued land before the CTA may exit (earlier ones were consumed)
            volatile int never = 0;
            for (int j = k_issued > kStages ? k_issued - kStages : 0; j < k_issued; ++j)
                ptx::mbar_wait(&bars[K_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, &never);
            for (int j = v_issued > kStages ? v_issued - kStages : 0; j < v_issued; ++j)
                ptx::mbar_wait(&bars[V_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, &never);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (whole warp)
        const uint64_t dq = gqp::sdesc(sbase + kOffQ, 16u, 1024u);
        const uint64_t dk0 = gqp::sdesc(sbase + kOffK, 16u, 1024u);
        const uint64_t dv0 = gqp::sdesc(sbase + kOffV, kBoxBytes, 1024u);
        bool ok = nt == 0 || ptx::mbar_wait(&bars[Q_READY], 0, abort);
        auto qk = [&](int j) -> bool {
            if (!ptx::mbar_wait(&bars[K_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, abort)) return false;
            ptx::tc_fence_after();
            const uint64_t dk = dk0 + (uint64_t)(((j & 1) * kTileBytes) >> 4);
            if (gqp::elect_one()) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint64_t koff = (uint64_t)(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4);
                    ptx::mma_ss(tmem + kColS + 128u * (j & 1), dq + koff, dk + koff, gqp::kIdescQK, k > 0);
                }
                ptx::mma_commit(&bars[S_FULL + (j & 1)]);
                ptx::mma_commit(&bars[K_EMPTY + (j & 1)]);
            }
            __syncwarp();
            return true;
        };
        auto pv = [&](int j) -> bool {
            if (!ptx::mbar_wait(&bars[V_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, abort)) return false;
            if (!ptx::mbar_wait(&bars[P_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, abort)) return false;
            ptx::tc_fence_after();
            const uint64_t dv = dv0 + (uint64_t)(((j & 1) * kTileBytes) >> 4);
            if (gqp::elect_one()) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    ptx::mma_ts(tmem + kColO, tmem + kColS + 128u * (j & 1) + 8u * k, dv + (uint64_t)(k * (2048 >> 4)),
                                gqp::kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
                ptx::mma_commit(&bars[V_EMPTY + (j & 1)]);
                ptx::mma_commit(&bars[O_READY]);
                if (j == nt - 1) ptx::mma_commit(&bars[O_FINAL]);
            }
            __syncwarp();
            return true;
        };
        if (ok && nt > 0) ok = qk(0);
        if (ok && nt > 1) ok = qk(1);
        for (int j = 0; j < nt && ok; ++j) {
            ok = pv(j);
            if (ok && j + 2 < nt) ok = qk(j + 2);
        }
        if (gqp::elect_one()) ptx::mma_commit(&bars[DRAIN]);
        __syncwarp();
        volatile int never = 0;
        ptx::mbar_wait(&bars[DRAIN], 0, &never);
    } else if (warp == 3) {
        // ------------------------------------------------------------ Q tile: rows = the group's heads
        // rows < group: bf16 of the rotated, scaled queries; the rest zero. Row r, 16-byte chunk c
        // (8 dims) sits in box c / 8 at row r, chunk (c % 8) ^ (r % 8) (the 128-byte swizzle).
        if (nt > 0) {
            for (int e = lane; e < kRows * 16; e += 32) {
                const int r = e >> 4, c = e & 15;
                uint4 w = make_uint4(0u, 0u, 0u, 0u);
                if (r < group) {
                    const float *src = q_rot + ((size_t)b * heads + h0 + r) * 128 + 8 * c;
                    const float4 a = *reinterpret_cast<const float4 *>(src);
                    const float4 d = *reinterpret_cast<const float4 *>(src + 4);
                    w = make_uint4(ptx::pack_bf16(a.x, a.y), ptx::pack_bf16(a.z, a.w), ptx::pack_bf16(d.x, d.y),
                                   ptx::pack_bf16(d.z, d.w));
                }
                *reinterpret_cast<uint4 *>(smem + kOffQ + (c >> 3) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = w;
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars[Q_READY]);
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------ softmax: lane g = head g
        const uint32_t trow = tmem;  // warp 4 reads TMEM lanes 0..31
        float m = -INFINITY, l = 0.f;  // running max (log2 units), sum of the weights
        bool done = nt > 0;
        for (int j = 0; j < nt; ++j) {
            if (!ptx::mbar_wait(&bars[S_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, abort)) { done = false; break; }
            ptx::tc_fence_after();
            const uint32_t cs = kColS + 128u * (j & 1);
            uint32_t v[128];
            gqp::tmem_ld128(trow + cs, v);
            ptx::tmem_ld_wait();
            const int valid = p1 - p0 - kRows * j;  // live positions in this tile (128 unless the last)
            if (valid < kRows) {
#pragma unroll
                for (int u = 0; u < 128; ++u)
                    if (u >= valid) v[u] = 0xff800000u;  // -inf
            }
            float mx0 = __uint_as_float(v[0]), mx1 = __uint_as_float(v[1]);
#pragma unroll
            for (int u = 2; u < 126; u += 4) {
                mx0 = gqp::max3(mx0, __uint_as_float(v[u]), __uint_as_float(v[u + 1]));
                mx1 = gqp::max3(mx1, __uint_as_float(v[u + 2]), __uint_as_float(v[u + 3]));
            }
            const float mnew =
                fmaxf(m, gqp::max3(mx0, mx1, fmaxf(__uint_as_float(v[126]), __uint_as_float(v[127]))) * gqp::kLog2eF);
            const bool raise = __any_sync(0xffffffffu, mnew > m + gqp::kRescaleMargin);
            float alpha = 1.f;
            if (raise) {
                alpha = ptx::ex2(m - mnew);  // 0 on the first tile
                l *= alpha;
                m = mnew;
            }
            l += gqp::p_half<0>(v, gqp::kLog2eF, m, trow + cs);
            l += gqp::p_half<1>(v, gqp::kLog2eF, m, trow + cs);
            if (raise && j > 0) {
                // O holds P V of tiles < j once the last of them has completed
                if (!ptx::mbar_wait(&bars[O_READY], (uint32_t)(j - 1) & 1u, abort)) { done = false; break; }
                ptx::tc_fence_after();
#pragma unroll 1
                for (int q = 0; q < 8; ++q) {
                    uint32_t a[16];
                    gqp::tmem_ld16(trow + kColO + 16u * q, a);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; ++u) a[u] = __float_as_uint(__uint_as_float(a[u]) * alpha);
                    ptx::tmem_st16(trow + kColO + 16u * q, a);
                }
            }
            if (valid < kRows) {
                // value rows past pos[b]: zero them (whole 128-byte rows of both boxes) once they landed
                if (!ptx::mbar_wait(&bars[V_FULL + (j & 1)], (uint32_t)(j >> 1) & 1u, abort)) { done = false; break; }
                uint8_t *vd = smem + kOffV + (j & 1) * kTileBytes;
                for (int e = valid * 16 + lane; e < kRows * 16; e += 32) {
                    const int r = e >> 4, c = e & 15;
                    *reinterpret_cast<uint4 *>(vd + (c >> 3) * kBoxBytes + r * 128 + ((c & 7) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bars[P_FULL + (j & 1)]);
        }
        if (done) done = ptx::mbar_wait(&bars[O_FINAL], 0, abort);
        const size_t ph = ((size_t)b * heads + h0 + lane) * splits + split;
        if (done) {
            ptx::tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t a[32];
                ptx::tmem_ld32(trow + kColO + 32u * q, a);
                ptx::tmem_ld_wait();
                if (lane < group) {
                    float4 *dst = reinterpret_cast<float4 *>(part_o + ph * 128 + 32 * q);
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        dst[u] = make_float4(__uint_as_float(a[4 * u]), __uint_as_float(a[4 * u + 1]),
                                             __uint_as_float(a[4 * u + 2]), __uint_as_float(a[4 * u + 3]));
                }
            }
            if (lane < group) {
                part_m[ph] = m * kLn2;  // natural units, as the combine expects
                part_l[ph] = l;
            }
        } else if (nt == 0 && lane < group) {
            // a chunk past pos[b] (or a bad position): nothing to merge
            part_m[ph] = -INFINITY;
            part_l[ph] = 0.f;
            for (int c = 0; c < 128; ++c) part_o[ph * 128 + c] = 0.f;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace gqd
}  // namespace la
