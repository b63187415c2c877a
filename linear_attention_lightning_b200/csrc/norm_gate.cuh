// Normalisation and gating of the attention output, after the intra- and
// inter-block outputs are summed ("MINIMAX SIGNAL LAB · M1", §03 Lightning
// Attention: the figure normalises and gates the sum; the pages print no
// formula). Reading: an RMS normalisation with a learned per-channel weight,
// then an elementwise sigmoid gate,
//   y[b][l][n] = gamma[n] * x[n] * rsqrt(mean_{group(n)} x^2 + eps) * sigmoid(g[b][l][n])
// over the token's channels n = h*dim + c, x[n] = o[b][h][l][c]; the mean runs
// over the head's dim channels (per_head) or over all heads*dim channels.
//
// Bound by HBM: o, g read and y written once. A persistent CTA per SM streams
// tiles of `tile` consecutive tokens of one batch through a kNgStages-deep TMA
// pipeline in shared memory: one 3-D box brings a tile's o for every head
// (o is [batch*heads][seq][dim]); two tiles stay in flight while the warps work
// on the third. The tile's gate rows, contiguous in g, are prefetched into L2 by
// one bulk copy when its o is requested, and read from there with 16-byte loads
// (a token's gate row is contiguous, as is its y row). The CTA's two groups of 256
// threads take alternate tokens of a tile, each on its own named barrier, so
// two tokens' reductions are in flight per SM. In a group each thread takes U
// 16-byte chunks of a token's row; a head's chunks sit in dim/E consecutive
// lanes of one warp (E values per chunk), so per-head sums are warp shuffles
// and per-token sums one group reduction (one barrier a token: the partial
// sums alternate between two buffers). y is written straight from registers
// with streaming stores (a token's row is contiguous in y).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace la {

constexpr int kNgThreads = 512;
constexpr int kNgGroup = 256;                   // threads per token group (two groups per CTA)
constexpr int kNgMaxChunks = 8;                 // heads*dim <= kNgGroup * kNgMaxChunks * (16 / sizeof(T))
constexpr int kNgStages = 3;
constexpr uint32_t kNgTileBytes = 65536;        // one tile of o at most
constexpr uint32_t kNgSmemBytes = kNgStages * kNgTileBytes + 64 + 128;

// Bulk prefetch of `bytes` contiguous bytes into L2 (address and size multiples of 16).
__device__ __forceinline__ void ng_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
                 : "memory");
}

template <typename T> struct NgVec;
template <> struct NgVec<float> {
    static constexpr int E = 4;
    __device__ static void unpack(const uint4 &w, float (&x)[8]) {
        x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
        x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
    }
    __device__ static uint4 pack(const float (&x)[8]) {
        return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
    }
};
template <> struct NgVec<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ static void unpack(const uint4 &w, float (&x)[8]) {
        const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(v[i] << 16);
            x[2 * i + 1] = __uint_as_float(v[i] & 0xffff0000u);
        }
    }
    __device__ static uint4 pack(const float (&x)[8]) {
        uint32_t v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 p = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            v[i] = *reinterpret_cast<const uint32_t *>(&p);
        }
        return make_uint4(v[0], v[1], v[2], v[3]);
    }
};

// tile: tokens per tile (tile * heads * dim * sizeof(T) <= kNgTileBytes).
template <typename T, int U>
__global__ void __launch_bounds__(kNgThreads, 1)
norm_gate_kernel(const __grid_constant__ CUtensorMap tm_o, const T *__restrict__ g,
                 const float *__restrict__ gamma, float eps, int batch, int heads, int seq, int dim, int per_head,
                 int tile, T *__restrict__ y) {
    using V = NgVec<T>;
    constexpr int E = V::E;
    extern __shared__ uint8_t ng_smem_raw[];
    const uint32_t raw = ptx::smem_addr(ng_smem_raw);
    uint8_t *smem = ng_smem_raw + (((raw + 127u) & ~127u) - raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kNgStages * kNgTileBytes);
    uint64_t *empty = full + kNgStages;
    int *abort_flag = reinterpret_cast<int *>(empty + kNgStages);

    const int n_ch = heads * dim, chunks = n_ch / E;
    const int lanes_per_head = dim / E;  // 8, 16 or 32: divides the warp
    const float inv_group = 1.f / (float)(per_head ? dim : n_ch);
    const uint32_t box_bytes = (uint32_t)tile * n_ch * sizeof(T);
    const int tiles_per_batch = (seq + tile - 1) / tile;
    const long long total = (long long)batch * tiles_per_batch;
    const int lane = threadIdx.x & 31;
    const int grp = threadIdx.x / kNgGroup, gtid = threadIdx.x % kNgGroup, gwarp = gtid >> 5;
    __shared__ float red[2][2][kNgGroup / 32];  // [group][buffer][warp]
    int nred = 0;                                // this group's reductions so far (picks the buffer)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNgStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], kNgThreads / 32);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_o);
    }
    __syncthreads();

    // tile `it` of this CTA (it = 0, 1, ...) is global tile blockIdx.x + it * gridDim.x
    auto issue = [&](long long it) {
        const long long gt = blockIdx.x + it * gridDim.x;
        if (gt >= total) return;
        const int s = (int)(it % kNgStages);
        if (it >= kNgStages && !ptx::mbar_wait(&empty[s], (uint32_t)((it / kNgStages - 1) & 1), abort_flag)) return;
        const int b = (int)(gt / tiles_per_batch), l0 = (int)(gt - (long long)b * tiles_per_batch) * tile;
        uint8_t *os = smem + s * kNgTileBytes;
        ptx::mbar_arrive_expect_tx(&full[s], box_bytes);
        ptx::tma_load_3d(os, &tm_o, &full[s], 0, l0, b * heads);
        ng_prefetch_l2(g + ((long long)b * seq + l0) * n_ch, (uint32_t)(min(tile, seq - l0) * n_ch * sizeof(T)));
    };
    if (threadIdx.x == 0)
        for (int it = 0; it < kNgStages - 1; ++it) issue(it);

    for (long long it = 0; blockIdx.x + it * gridDim.x < total; ++it) {
        if (threadIdx.x == 0) issue(it + kNgStages - 1);
        const int s = (int)(it % kNgStages);
        if (!ptx::mbar_wait(&full[s], (uint32_t)((it / kNgStages) & 1), abort_flag)) break;
        const long long gt = blockIdx.x + it * gridDim.x;
        const int b = (int)(gt / tiles_per_batch), l0 = (int)(gt - (long long)b * tiles_per_batch) * tile;
        const int tcount = min(tile, seq - l0);
        const T *os = reinterpret_cast<const T *>(smem + s * kNgTileBytes);
        for (int t = grp; t < tcount; t += 2) {
            // the token's gate chunks first, so that their loads (from L2) overlap the
            // sums; at U = 8 (16-bit) they are loaded where used, to stay in registers
            constexpr bool kEarlyGate = U * E <= 32;
            const T *grow = g + ((long long)b * seq + l0 + t) * n_ch;
            uint4 gw[U];
            if (kEarlyGate) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int k = gtid + kNgGroup * u;
                    if (k < chunks) gw[u] = __ldcs(reinterpret_cast<const uint4 *>(grow + k * E));
                }
            }
            float x[U][8], ss[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = gtid + kNgGroup * u;
                ss[u] = 0.f;
                if (k < chunks) {
                    const int n0 = k * E, h = n0 / dim, c0 = n0 - h * dim;
                    V::unpack(*reinterpret_cast<const uint4 *>(os + ((size_t)h * tile + t) * dim + c0), x[u]);
#pragma unroll
                    for (int e = 0; e < E; ++e) ss[u] += x[u][e] * x[u][e];
                }
            }
            if (per_head) {
#pragma unroll
                for (int u = 0; u < U; ++u)
                    for (int off = 1; off < lanes_per_head; off <<= 1) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
            } else {
                float tsum = 0.f;
#pragma unroll
                for (int u = 0; u < U; ++u) tsum += ss[u];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) tsum += __shfl_xor_sync(0xffffffffu, tsum, off);
                // buffers alternate over the group's tokens: a group's next write to one
                // follows its next barrier, which every thread reaches only after reading it
                float *rb = red[grp][nred & 1];
                ++nred;
                if (lane == 0) rb[gwarp] = tsum;
                ptx::named_bar_sync(1 + grp, kNgGroup);
                float all = 0.f;
#pragma unroll
                for (int w = 0; w < kNgGroup / 32; ++w) all += rb[w];
#pragma unroll
                for (int u = 0; u < U; ++u) ss[u] = all;
            }
            T *yrow = y + ((long long)b * seq + l0 + t) * n_ch;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = gtid + kNgGroup * u;
                if (k < chunks) {
                    const int n0 = k * E;
                    const float inv = rsqrtf(ss[u] * inv_group + eps);
                    float gv[8], out[8];
                    V::unpack(kEarlyGate ? gw[u] : __ldcs(reinterpret_cast<const uint4 *>(grow + n0)), gv);
                    float gm[8];
#pragma unroll
                    for (int e = 0; e < E; e += 4) {
                        const float4 g4 = __ldg(reinterpret_cast<const float4 *>(gamma + n0 + e));
                        gm[e] = g4.x; gm[e + 1] = g4.y; gm[e + 2] = g4.z; gm[e + 3] = g4.w;
                    }
                    if (sizeof(T) == 2) {
                        // bf16: sigmoid(g) = 1/2 + tanh(g/2)/2 with the SFU's tanh (one SFU op)
#pragma unroll
                        for (int e = 0; e < E; ++e) {
                            float th;
                            asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(0.5f * gv[e]));
                            out[e] = gm[e] * x[u][e] * inv * fmaf(0.5f, th, 0.5f);
                        }
                    } else {
                        // sigmoid with the fast divide: a few ulp, far inside the output's rounding
#pragma unroll
                        for (int e = 0; e < E; ++e) out[e] = __fdividef(gm[e] * x[u][e] * inv, 1.f + __expf(-gv[e]));
                    }
                    __stcs(reinterpret_cast<uint4 *>(yrow + n0), V::pack(out));
                }
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[s]);
    }
    // copies issued for tiles past the end of this CTA's work were never issued
    // (issue() skips them), so nothing is in flight here
}

}  // namespace la
