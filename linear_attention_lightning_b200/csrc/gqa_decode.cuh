// One decode step of the softmax attention layer that M1 places after every
// seven Lightning layers ("MINIMAX SIGNAL LAB · M1", §02: 64 query heads x 128,
// softmax K/V 8 x 128, RoPE on 64 of the 128 dims in the softmax layers only;
// §04: those layers keep a bf16 KV cache that grows with the context).
// Readings (the pages print no formula): grouped-query attention, query head h
// reads KV head h / (heads / kv_heads); scores scaled by `scale`; rotate-half
// RoPE on the first `rot` dims with theta_i = base^{-2i/rot}; the cache holds
// rotated keys. Per sequence b the new token sits at position pos[b]:
//   o = sum_{p <= pos} softmax_p(scale * rope(q) . k_p) v_p.
//
// Split over the context (the step reads the whole cache once and is bound by
// HBM): gqa_append writes the new rotated key and value into the cache;
// gqa_append also rotates and scales the queries once; gqa_partial gives each
// CTA a chunk of kGqaChunk positions of one (sequence, KV head) for all heads
// of the group and leaves a partial softmax (running max, sum, weighted
// values) in the workspace; gqa_combine merges the chunks.
// Rotation angles are taken in double: pos * theta reaches 1e5 radians.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace la {

constexpr int kGqaThreads = 256;
constexpr int kGqaChunk = 2048;        // positions per CTA
constexpr int kGqaDim = 128;
constexpr int kGqaMaxGroup = 8;        // query heads per KV head

template <typename T> __device__ __forceinline__ void gqa_store(T *p, float x);
template <> __device__ __forceinline__ void gqa_store<float>(float *p, float x) { *p = x; }
template <> __device__ __forceinline__ void gqa_store<__nv_bfloat16>(__nv_bfloat16 *p, float x) {
    *p = __float2bfloat16_rn(x);
}

// rotate-half RoPE of element c of a head (dim kGqaDim) given the head in x[]
__device__ __forceinline__ float gqa_rope_elem(const float *x, int c, int rot, double base, int pos) {
    const int half = rot / 2;
    if (c >= rot) return x[c];
    const int i = c < half ? c : c - half;
    double sn, cs;
    sincos((double)pos * pow(base, -2.0 * i / (double)rot), &sn, &cs);
    return c < half ? (float)((double)x[c] * cs - (double)x[c + half] * sn)
                    : (float)((double)x[c] * cs + (double)x[c - half] * sn);
}

// grid (batch, kv_heads), kGqaDim threads: cache[b][hk][pos] <- rope(k_new),
// v_new; and the group's queries rotated and scaled once, in fp32, for every
// chunk of the partial kernel: q_rot [batch][heads][kGqaDim].
template <typename T>
__global__ void __launch_bounds__(kGqaDim)
gqa_append_kernel(const T *__restrict__ q, const T *__restrict__ k_new, const T *__restrict__ v_new, T *k_cache,
                  T *v_cache, const int *__restrict__ pos, int heads, int kv_heads, int cap, int rot, double base,
                  float scale, float *__restrict__ q_rot) {
    __shared__ float kx[kGqaDim];
    const int b = blockIdx.x, hk = blockIdx.y, c = threadIdx.x;
    const size_t kv = (size_t)b * kv_heads + hk;
    const int p = pos[b];
    if (p < 0 || p >= cap) {  // never write outside the cache
        if (c == 0) atomicOr(&g_device_status, kBadDeviceArgFlag);
        return;
    }
    kx[c] = to_f32(k_new[kv * kGqaDim + c]);
    __syncthreads();
    const size_t at = (kv * cap + p) * kGqaDim + c;
    k_cache[at] = from_f32<T>(gqa_rope_elem(kx, c, rot, base, p));
    v_cache[at] = v_new[kv * kGqaDim + c];
    const int group = heads / kv_heads;
    for (int g = 0; g < group; ++g) {
        const size_t hq = (size_t)b * heads + hk * group + g;
        __syncthreads();
        kx[c] = to_f32(q[hq * kGqaDim + c]);
        __syncthreads();
        q_rot[hq * kGqaDim + c] = scale * gqa_rope_elem(kx, c, rot, base, p);
    }
}

constexpr int kGqaStages = 3;
constexpr uint32_t kGqaBoxRowBytes = 128;      // TMA box width: 128 bytes, 128B-swizzled
constexpr uint32_t kGqaTileBytes = 16384;      // one tile of K (or V): TILE rows x kGqaDim elements
constexpr uint32_t kGqaSmemBytes = kGqaStages * 2 * kGqaTileBytes + 1024 + 64;

// byte offset of 16-byte chunk c (of kGqaDim * sizeof(T) / 16) of row r in a staged tile:
// 128-byte boxes side by side, each [TILE rows][128 B] with the 128B swizzle
template <int TILE>
__device__ __forceinline__ uint32_t gqa_chunk_off(int r, int c) {
    return (uint32_t)(c >> 3) * TILE * kGqaBoxRowBytes + (uint32_t)r * kGqaBoxRowBytes +
           (uint32_t)(((c & 7) ^ (r & 7)) << 4);
}

// grid (splits, kv_heads, batch). Partial softmax of chunk `split` for the
// group's query heads: part_m / part_l [batch][heads][splits],
// part_o [batch][heads][splits][kGqaDim]. K and V tiles of TILE positions
// (64 bf16 / 32 f32 rows = 16 KB) stream in through a kGqaStages-deep TMA
// pipeline; per tile:
//   scores  SL adjacent lanes share a position; lane slice s takes the
//           16-byte chunks s, s + SL, ... of the row for all heads of the
//           group (the swizzle keeps the reads off each other's banks), and
//           the slices meet in a shuffle;
//   softmax warp g keeps head g's running max and sum and turns the tile's
//           scores into weights (stored position-major);
//   P.V     warp w takes positions w, w + 8, ...; lane l holds dims
//           4l .. 4l+3 of every head, so one value load serves all heads.
// Rows past the chunk's last position are never read into a sum: the cache
// beyond pos[b] may hold anything. The warps' partial sums meet once, after
// the last tile, in the stage buffers.
template <typename T>
__global__ void __launch_bounds__(kGqaThreads)
gqa_partial_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const float *__restrict__ q_rot, const int *__restrict__ pos, int heads, int kv_heads, int cap,
                   int splits, float *__restrict__ part_m, float *__restrict__ part_l, float *__restrict__ part_o) {
    constexpr int G = kGqaMaxGroup;
    constexpr int EV = 16 / (int)sizeof(T);               // elements per 16-byte chunk
    constexpr int TILE = (int)(kGqaTileBytes / (kGqaDim * sizeof(T)));  // 64 or 32
    constexpr int SL = kGqaThreads / TILE;                // lanes per position in the score pass: 4 or 8
    constexpr int CPR = kGqaDim / EV;                     // 16-byte chunks per row: 16 or 32
    constexpr int CPS = CPR / SL;                         // chunks per lane: 4
    constexpr int WARPS = kGqaThreads / 32;
    constexpr int PPW = TILE / WARPS;                     // positions per warp in P.V: 8 or 4
    constexpr int NPL = TILE / 32;                        // scores per lane in the softmax pass
    constexpr int NBOX = (int)(kGqaDim * sizeof(T) / kGqaBoxRowBytes);  // boxes per tile: 2 or 4
    static_assert(kGqaStages * 2 * kGqaTileBytes >= sizeof(float) * WARPS * G * kGqaDim, "reduction fits");
    __shared__ __align__(16) float qs[G][kGqaDim];
    __shared__ __align__(16) float scs[G][TILE];
    __shared__ __align__(16) float wt[TILE][G];
    __shared__ float corr_s[G];
    __shared__ uint64_t full[kGqaStages], empty[kGqaStages];
    __shared__ int abort_flag;
    extern __shared__ uint8_t gqa_smem_raw[];
    const uint32_t raw = ptx::smem_addr(gqa_smem_raw);
    uint8_t *stage0 = gqa_smem_raw + (((raw + 1023u) & ~1023u) - raw);  // 128B swizzle: 1024-aligned

    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int group = heads / kv_heads;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int P = pos[b];
    const bool bad = P < 0 || P >= cap;  // recorded by the append kernel; read nothing then
    const int p0 = split * kGqaChunk, p1 = bad ? p0 : min(p0 + kGqaChunk, P + 1);
    const int ntiles = p1 > p0 ? (p1 - p0 + TILE - 1) / TILE : 0;
    const long long row0 = ((long long)b * kv_heads + hk) * cap + p0;  // tensor row of position p0
    const int h0 = hk * group;

    if (tid == 0) {
        for (int st = 0; st < kGqaStages; ++st) {
            ptx::mbar_init(&full[st], 1);
            ptx::mbar_init(&empty[st], WARPS);
        }
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    for (int e = tid; e < G * kGqaDim / 4; e += kGqaThreads) {
        const int g = e / (kGqaDim / 4);
        reinterpret_cast<float4 *>(&qs[0][0])[e] =
            g < group ? reinterpret_cast<const float4 *>(q_rot + ((size_t)b * heads + h0) * kGqaDim)[e]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    auto issue = [&](int it) {
        if (it >= ntiles) return;
        const int st = it % kGqaStages;
        if (it >= kGqaStages && !ptx::mbar_wait(&empty[st], (uint32_t)((it / kGqaStages - 1) & 1), &abort_flag))
            return;
        uint8_t *kd = stage0 + st * 2 * kGqaTileBytes;
        ptx::mbar_arrive_expect_tx(&full[st], 2 * kGqaTileBytes);
        const int y = (int)(row0 + (long long)it * TILE);
        for (int bx = 0; bx < NBOX; ++bx) {
            const int x = bx * (int)(kGqaBoxRowBytes / sizeof(T));
            ptx::tma_load_2d(kd + bx * TILE * kGqaBoxRowBytes, &tm_k, &full[st], x, y);
            ptx::tma_load_2d(kd + kGqaTileBytes + bx * TILE * kGqaBoxRowBytes, &tm_v, &full[st], x, y);
        }
    };
    if (tid == 0)
        for (int it = 0; it < kGqaStages - 1; ++it) issue(it);

    float m_run = -INFINITY, l_run = 0.f;   // head `warp`'s statistics (warps < group)
    float acc[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[g][u] = 0.f;
    for (int it = 0; it < ntiles; ++it) {
        if (tid == 0) issue(it + kGqaStages - 1);
        const int st = it % kGqaStages;
        if (!ptx::mbar_wait(&full[st], (uint32_t)((it / kGqaStages) & 1), &abort_flag)) break;
        const uint8_t *ks = stage0 + st * 2 * kGqaTileBytes, *vs = ks + kGqaTileBytes;
        const int rows = min(TILE, p1 - p0 - it * TILE);
        // scores of position r: lane slice sl takes chunks sl, sl + SL, ... for every head
        {
            const int r = tid / SL, sl = tid % SL;
            float2 dot2[G];  // even and odd dims accumulate side by side
#pragma unroll
            for (int g = 0; g < G; ++g) dot2[g] = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < CPS; ++j) {
                const int c = sl + SL * j;
                const uint4 w = *reinterpret_cast<const uint4 *>(ks + gqa_chunk_off<TILE>(r, c));
                const T *kt = reinterpret_cast<const T *>(&w);
                float kf[EV];
#pragma unroll
                for (int e = 0; e < EV; ++e) kf[e] = to_f32(kt[e]);
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e4 = 0; e4 < EV; e4 += 4) {
                        const float4 qv = *reinterpret_cast<const float4 *>(&qs[g][c * EV + e4]);
                        dot2[g] = ptx::fma2(make_float2(qv.x, qv.y), make_float2(kf[e4], kf[e4 + 1]), dot2[g]);
                        dot2[g] = ptx::fma2(make_float2(qv.z, qv.w), make_float2(kf[e4 + 2], kf[e4 + 3]), dot2[g]);
                    }
            }
            float dot[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                dot[g] = dot2[g].x + dot2[g].y;
#pragma unroll
                for (int off = 1; off < SL; off <<= 1) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], off);
            }
            if (sl == 0)
#pragma unroll
                for (int g = 0; g < G; ++g) scs[g][r] = dot[g];
        }
        __syncthreads();
        // softmax statistics: warp g owns head g
        if (warp < group) {
            float sv[NPL];
            float mt = -INFINITY;
#pragma unroll
            for (int i = 0; i < NPL; ++i) {
                const int r = lane + 32 * i;
                sv[i] = r < rows ? scs[warp][r] : -INFINITY;
                mt = fmaxf(mt, sv[i]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float m_new = fmaxf(m_run, mt);
            const float corr = __expf(m_run - m_new);  // 0 on the first tile (m_run = -inf)
            float ws = 0.f;
#pragma unroll
            for (int i = 0; i < NPL; ++i) {
                const float w = __expf(sv[i] - m_new);
                wt[lane + 32 * i][warp] = w;
                ws += w;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
            l_run = l_run * corr + ws;
            m_run = m_new;
            if (lane == 0) corr_s[warp] = corr;
        } else if (warp < G) {
#pragma unroll
            for (int i = 0; i < NPL; ++i) wt[lane + 32 * i][warp] = 0.f;  // heads past the group weigh nothing
            if (lane == 0) corr_s[warp] = 1.f;
        }
        __syncthreads();
        // P.V: positions warp, warp + WARPS, ...; lane: dims 4 lane .. 4 lane + 3 of every head
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float cg = corr_s[g];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[g][u] *= cg;
        }
#pragma unroll
        for (int j = 0; j < PPW; ++j) {
            const int r = warp + WARPS * j;
            if (r >= rows) break;  // uniform in the warp
            const int c = 4 * lane / EV, within = 4 * lane % EV;  // 4 values inside one 16-byte chunk
            const T *vrow = reinterpret_cast<const T *>(vs + gqa_chunk_off<TILE>(r, c)) + within;
            float vf[4];
            if (sizeof(T) == 2) {  // four bf16 in one 8-byte load
                const uint2 rawv = *reinterpret_cast<const uint2 *>(vrow);
                vf[0] = __uint_as_float(rawv.x << 16); vf[1] = __uint_as_float(rawv.x & 0xffff0000u);
                vf[2] = __uint_as_float(rawv.y << 16); vf[3] = __uint_as_float(rawv.y & 0xffff0000u);
            } else {
                const float4 rawv = *reinterpret_cast<const float4 *>(vrow);
                vf[0] = rawv.x; vf[1] = rawv.y; vf[2] = rawv.z; vf[3] = rawv.w;
            }
            const float4 wa = *reinterpret_cast<const float4 *>(&wt[r][0]);
            const float4 wb = *reinterpret_cast<const float4 *>(&wt[r][4]);
            const float wv[G] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float2 lo = ptx::fma2(make_float2(wv[g], wv[g]), make_float2(vf[0], vf[1]),
                                           make_float2(acc[g][0], acc[g][1]));
                const float2 hi = ptx::fma2(make_float2(wv[g], wv[g]), make_float2(vf[2], vf[3]),
                                           make_float2(acc[g][2], acc[g][3]));
                acc[g][0] = lo.x; acc[g][1] = lo.y; acc[g][2] = hi.x; acc[g][3] = hi.y;
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[st]);
        __syncthreads();  // scs / wt are rewritten for the next tile
    }
    // the warps' partial sums meet in the stage buffers (every issued copy has landed and been used)
    __syncthreads();
    float *red = reinterpret_cast<float *>(stage0);  // WARPS x G x kGqaDim floats
#pragma unroll
    for (int g = 0; g < G; ++g)
        *reinterpret_cast<float4 *>(&red[((size_t)warp * G + g) * kGqaDim + 4 * lane]) =
            make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    if (warp < group && lane == 0) {
        const size_t ph = ((size_t)b * heads + h0 + warp) * splits + split;
        part_m[ph] = m_run;  // -inf for a chunk past pos[b]
        part_l[ph] = l_run;
    }
    __syncthreads();
    for (int e = tid; e < group * kGqaDim; e += kGqaThreads) {
        const int g = e / kGqaDim, c = e % kGqaDim;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) sum += red[((size_t)w * G + g) * kGqaDim + c];
        part_o[(((size_t)b * heads + h0 + g) * splits + split) * kGqaDim + c] = sum;
    }
}

// grid (batch * heads), kGqaDim threads: merge the chunks of one query head
template <typename T>
__global__ void __launch_bounds__(kGqaDim)
gqa_combine_kernel(const float *__restrict__ part_m, const float *__restrict__ part_l,
                   const float *__restrict__ part_o, int splits, T *__restrict__ o) {
    const size_t bh = blockIdx.x;
    const int c = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part_m[bh * splits + s]);
    float num = 0.f, den = 0.f;
    for (int s = 0; s < splits; ++s) {
        const float m = part_m[bh * splits + s];
        if (m == -INFINITY) continue;  // a chunk past pos[b]
        const float w = __expf(m - M);
        den += w * part_l[bh * splits + s];
        num += w * part_o[(bh * splits + s) * kGqaDim + c];
    }
    gqa_store<T>(o + bh * kGqaDim + c, den > 0.f ? num / den : 0.f);  // den = 0 only for a bad position
}

}  // namespace la
