// Shared device helpers for the Lightning Attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la {

// Status word: kernels set LA_ERR_TIMEOUT here when a bounded wait gives up,
// and kBadDeviceArgFlag when they meet an out-of-range device-side argument.
// It lives in managed memory, one word for the process, so that the host can
// read it without synchronising anything: every launching entry point looks
// at it before it launches, and lightning_last_device_status() reads it after
// synchronising a stream. Kernels of every device and stream share it.
__managed__ unsigned int g_device_status;
// flag in the status word: a kernel met an out-of-range device-side argument
// (a decode position outside the cache) and skipped the work it governs
constexpr unsigned int kBadDeviceArgFlag = 1u;

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// e^{-s * n} for n >= 0 through exp2f; s is the per-head slope.
__device__ __forceinline__ float decay_pow(float s, float n) { return exp2f(-s * kLog2e * n); }

// State snapshots for a prefix cache: the fp32 state after every `interval`
// tokens (a multiple of the block), `count` = seq / interval of them per
// (batch, head), laid out [batch*heads][count][dim][dim]. ptr == nullptr: none.
struct Snapshots {
    float *ptr;
    int interval;
    int count;
};

// Where the state after the first `tokens_done` tokens of (batch*heads index)
// bh goes, or nullptr when that position takes no snapshot.
__device__ __forceinline__ float *snapshot_at(const Snapshots &sn, size_t bh, int tokens_done, int dim) {
    if (sn.ptr == nullptr || tokens_done <= 0 || tokens_done % sn.interval != 0) return nullptr;
    const int n = tokens_done / sn.interval - 1;
    if (n >= sn.count) return nullptr;
    return sn.ptr + ((size_t)bh * sn.count + n) * dim * dim;
}

}  // namespace la
