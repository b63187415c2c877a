// liblightning.so: host side of the C ABI declared in include/lightning.h.
//
// Argument checking happens here, before any launch; every check failure
// returns a status and records a message for lightning_last_error_message().
// The library allocates nothing: all tensors, and the workspace (the range
// guard's per-head records of the tensor-core prefill), belong to the caller.
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/lightning.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_simt.cuh"
#include "gqa_decode.cuh"
#include "gqa_prefill.cuh"
#include "gqa_decode_tc.cuh"
#include "selftest.cuh"
#include "norm_gate.cuh"
#include "prefill_pair.cuh"
#include "prefill_tc.cuh"

namespace {

thread_local std::string g_last_error;

la_status fail(la_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

la_status ok() {
    g_last_error.clear();
    return LA_OK;
}

la_status cuda_fail(cudaError_t e, const char *what) {
    return fail(LA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// The status a kernel recorded in the status word, as an la_status (LA_OK for 0).
la_status status_of_word(unsigned int word) {
    if (word & LA_ERR_TIMEOUT)
        return fail(LA_ERR_TIMEOUT, "a device-side wait of an earlier kernel gave up (status word 0x%x)", word);
    if (word & la::kBadDeviceArgFlag)
        return fail(LA_ERR_INVALID_ARG,
                    "an earlier kernel met an out-of-range device-side argument (status word 0x%x)", word);
    return LA_OK;
}

// Called by every entry point just before its first launch (never on a path
// that launches nothing, so that host-only calls need no CUDA context): a
// failure an earlier kernel recorded is returned now, the word is cleared, and
// nothing is launched. The word is read without any synchronisation; a kernel
// still running may record a failure after this look, and the next call sees it.
la_status earlier_failure() {
    if (__atomic_load_n(&la::g_device_status, __ATOMIC_ACQUIRE) == 0u) return LA_OK;
    return status_of_word(__atomic_exchange_n(&la::g_device_status, 0u, __ATOMIC_ACQ_REL));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void *p, size_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return {a, a + bytes};
}

bool overlaps(Range a, Range b) {
    return a.lo < a.hi && b.lo < b.hi && a.lo < b.hi && b.lo < a.hi;
}

size_t elem_bytes(la_dtype dt) { return dt == LA_DTYPE_BF16 ? 2 : 4; }

struct PrefillArgs {
    const void *q, *k, *v;
    la_dtype dtype;
    const float *slopes;
    int batch, heads, seq, dim, block;
    const float *state_in;
    void *o;
    float *state_out;
    la::Snapshots sn;  // prefix-cache snapshots; sn.ptr == nullptr: none
    void *workspace;
    size_t workspace_bytes;
};

// Workspace a prefill request needs: the range guard's records for the CTA-pair
// kernel, none for the others.
size_t prefill_workspace_bytes(int batch, int heads, int variant) {
    if (variant == LA_VARIANT_TCGEN05_PAIR) return la::pair_workspace_bytes((long long)batch * heads);
    if (variant == LA_VARIANT_TCGEN05) return la::tc_workspace_bytes((long long)batch * heads);
    return 0;
}

// A workspace of at least `need` bytes, 16-byte aligned, overlapping none of `others`.
la_status check_workspace(const void *ws, size_t bytes, size_t need, const Range *others, int n_others) {
    if (need == 0) return LA_OK;
    if (!ws || bytes < need)
        return fail(LA_ERR_INVALID_ARG, "this call needs %zu bytes of workspace (got %zu)", need, ws ? bytes : (size_t)0);
    if (!aligned16(ws)) return fail(LA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    const Range rw = range_of(ws, need);
    for (int i = 0; i < n_others; ++i)
        if (overlaps(rw, others[i])) return fail(LA_ERR_INVALID_ARG, "workspace overlaps an input or an output");
    return LA_OK;
}

// Shape / dtype checks shared by the launcher and the variant query.
la_status check_prefill_shape(la_dtype dtype, int batch, int heads, int seq, int dim, int block) {
    if (dtype != LA_DTYPE_F32 && dtype != LA_DTYPE_BF16)
        return fail(LA_ERR_INVALID_ARG, "dtype %d is neither LA_DTYPE_F32 nor LA_DTYPE_BF16", (int)dtype);
    if (batch < 0 || heads < 1 || seq < 0)
        return fail(LA_ERR_INVALID_ARG, "need batch >= 0, heads >= 1, seq >= 0 (got %d, %d, %d)",
                    batch, heads, seq);
    if (block < 1) return fail(LA_ERR_INVALID_ARG, "block must be >= 1 (got %d)", block);
    if (dim != 64 && dim != 128)
        return fail(LA_ERR_UNSUPPORTED, "dim %d unsupported (64 or 128)", dim);
    if ((long long)batch * heads > (1ll << 28))
        return fail(LA_ERR_UNSUPPORTED, "batch*heads too large (at most 2^28)");
    return LA_OK;
}

int choose_variant(la_dtype dtype, int dim, int block, int requested) {
    const bool bf16 = dtype == LA_DTYPE_BF16;
    const bool tc_ok = la::tc_supports(bf16, dim, block);
    const bool pair_ok = la::pair_supports(bf16, dim, block);
    switch (requested) {
        case LA_VARIANT_AUTO:
            return pair_ok ? LA_VARIANT_TCGEN05_PAIR : (tc_ok ? LA_VARIANT_TCGEN05 : LA_VARIANT_SIMT);
        case LA_VARIANT_SIMT: return LA_VARIANT_SIMT;
        case LA_VARIANT_TCGEN05: return tc_ok ? LA_VARIANT_TCGEN05 : -1;
        case LA_VARIANT_TCGEN05_PAIR: return pair_ok ? LA_VARIANT_TCGEN05_PAIR : -1;
        default: return -1;
    }
}

la_status check_prefill_pointers(const PrefillArgs &a) {
    const size_t eb = elem_bytes(a.dtype);
    const size_t n_tok = (size_t)a.batch * a.heads * a.seq * a.dim;
    const size_t n_state = (size_t)a.batch * a.heads * a.dim * a.dim;
    if (a.seq > 0 && (!a.q || !a.k || !a.v || !a.o))
        return fail(LA_ERR_INVALID_ARG, "q, k, v and o must be non-NULL when seq > 0");
    if (!a.slopes) return fail(LA_ERR_INVALID_ARG, "slopes must be non-NULL");
    const void *ptrs[] = {a.q, a.k, a.v, a.o, a.slopes, a.state_in, a.state_out};
    const char *names[] = {"q", "k", "v", "o", "slopes", "state_in", "state_out"};
    for (int i = 0; i < 7; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(LA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    const Range ro = range_of(a.o, a.seq > 0 ? n_tok * eb : 0);
    const Range rin[] = {range_of(a.q, n_tok * eb), range_of(a.k, n_tok * eb),
                         range_of(a.v, n_tok * eb), range_of(a.slopes, sizeof(float) * a.heads),
                         range_of(a.state_in, a.state_in ? n_state * 4 : 0),
                         range_of(a.state_out, a.state_out ? n_state * 4 : 0)};
    for (const Range &r : rin)
        if (overlaps(ro, r)) return fail(LA_ERR_INVALID_ARG, "o overlaps an input or a state");
    if (a.state_out) {
        const Range rs = range_of(a.state_out, n_state * 4);
        for (int i = 0; i < 4; ++i)
            if (overlaps(rs, rin[i])) return fail(LA_ERR_INVALID_ARG, "state_out overlaps an input");
        if (a.state_in && a.state_in != a.state_out && overlaps(rs, rin[4]))
            return fail(LA_ERR_INVALID_ARG, "state_out partially overlaps state_in");
    }
    return LA_OK;
}

// Snapshot interval and buffer: checked after check_prefill_pointers.
la_status check_snapshots(const PrefillArgs &a) {
    if (a.sn.interval < a.block || a.sn.interval % a.block != 0)
        return fail(LA_ERR_INVALID_ARG, "snapshot interval %d must be a positive multiple of block %d",
                    a.sn.interval, a.block);
    if (a.sn.count == 0) return LA_OK;
    if (!a.sn.ptr) return fail(LA_ERR_INVALID_ARG, "snapshots must be non-NULL when seq / interval > 0");
    if (!aligned16(a.sn.ptr)) return fail(LA_ERR_INVALID_ARG, "snapshots is not 16-byte aligned");
    const size_t eb = elem_bytes(a.dtype);
    const size_t n_tok = (size_t)a.batch * a.heads * a.seq * a.dim;
    const size_t n_state = (size_t)a.batch * a.heads * a.dim * a.dim;
    const Range rs = range_of(a.sn.ptr, n_state * (size_t)a.sn.count * sizeof(float));
    const Range others[] = {range_of(a.q, n_tok * eb), range_of(a.k, n_tok * eb), range_of(a.v, n_tok * eb),
                            range_of(a.o, n_tok * eb), range_of(a.slopes, sizeof(float) * a.heads),
                            range_of(a.state_in, a.state_in ? n_state * 4 : 0),
                            range_of(a.state_out, a.state_out ? n_state * 4 : 0)};
    for (const Range &r : others)
        if (overlaps(rs, r)) return fail(LA_ERR_INVALID_ARG, "snapshots overlaps an input, o or a state");
    return LA_OK;
}

// The workspace of a prefill request (after check_prefill_pointers and, for
// snapshots, check_snapshots).
la_status check_prefill_workspace(const PrefillArgs &a, int variant) {
    if (a.batch == 0 || a.seq == 0) return LA_OK;
    const size_t eb = elem_bytes(a.dtype);
    const size_t n_tok = (size_t)a.batch * a.heads * a.seq * a.dim;
    const size_t n_state = (size_t)a.batch * a.heads * a.dim * a.dim;
    const Range others[] = {range_of(a.q, n_tok * eb), range_of(a.k, n_tok * eb), range_of(a.v, n_tok * eb),
                            range_of(a.o, n_tok * eb), range_of(a.slopes, sizeof(float) * a.heads),
                            range_of(a.state_in, a.state_in ? n_state * 4 : 0),
                            range_of(a.state_out, a.state_out ? n_state * 4 : 0),
                            range_of(a.sn.ptr, a.sn.ptr ? n_state * (size_t)a.sn.count * 4 : 0)};
    return check_workspace(a.workspace, a.workspace_bytes, prefill_workspace_bytes(a.batch, a.heads, variant), others,
                           8);
}

template <typename T, int D>
la_status launch_simt(const PrefillArgs &a, cudaStream_t stream) {
    auto kern = la::prefill_simt_kernel<T, D>;
    const size_t smem = la::simt_smem_bytes<D>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill_simt)");
    dim3 grid((unsigned)((size_t)a.batch * a.heads * (D / la::kSimtCols)));
    kern<<<grid, la::kSimtThreads, smem, stream>>>(
        static_cast<const T *>(a.q), static_cast<const T *>(a.k), static_cast<const T *>(a.v),
        a.slopes, a.heads, a.seq, a.block, a.state_in, static_cast<T *>(a.o), a.state_out, a.sn,
        la::SimtPass{0, 0, 0, 0});
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefill_simt launch");
    return ok();
}

struct NgArgs {
    const void *o, *gate;
    const float *gamma;
    float eps;
    int batch, heads, seq, dim, per_head;
    void *y;
    long long tokens;
    cudaStream_t stream;
};

// 3-D tensor map without swizzle over a tensor of 16- or 32-bit elements.
bool make_plain_map(CUtensorMap *map, const void *base, bool bf16, const cuuint64_t (&dims)[3],
                    const cuuint64_t (&strides)[2], const cuuint32_t (&box)[3], std::string *err) {
    auto fn = la::tc::encode_fn(err);
    if (!fn) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = "cuTensorMapEncodeTiled failed (CUresult " + std::to_string((int)r) + ")";
        return false;
    }
    return true;
}

template <typename T, int U>
la_status launch_norm_gate(const NgArgs &a) {
    const size_t eb = sizeof(T);
    const long long n_ch = (long long)a.heads * a.dim;
    long long tile = (long long)la::kNgTileBytes / (n_ch * (long long)eb);
    tile = tile < 1 ? 1 : (tile > 64 ? 64 : tile);
    const bool bf16 = sizeof(T) == 2;
    CUtensorMap mo;
    // o: [batch*heads][seq][dim], box = one tile of tokens for every head of a batch
    const cuuint64_t odims[3] = {(cuuint64_t)a.dim, (cuuint64_t)a.seq, (cuuint64_t)a.batch * a.heads};
    const cuuint64_t ostr[2] = {(cuuint64_t)a.dim * eb, (cuuint64_t)a.seq * a.dim * eb};
    const cuuint32_t obox[3] = {(cuuint32_t)a.dim, (cuuint32_t)tile, (cuuint32_t)a.heads};
    if (!make_plain_map(&mo, a.o, bf16, odims, ostr, obox, &g_last_error)) return LA_ERR_CUDA;
    auto kern = la::norm_gate_kernel<T, U>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)la::kNgSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(norm_gate)");
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long tiles = (long long)a.batch * ((a.seq + tile - 1) / tile);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    kern<<<grid, la::kNgThreads, la::kNgSmemBytes, a.stream>>>(mo, static_cast<const T *>(a.gate), a.gamma, a.eps,
                                                              a.batch, a.heads, a.seq, a.dim, a.per_head, (int)tile,
                                                              static_cast<T *>(a.y));
    e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "norm_gate launch");
}

// Workspace of one GQA decode step: per (sequence, query head, chunk) the
// running max, the sum and the weighted values of the chunk's softmax.
struct GqaLayout {
    int splits;
    size_t m_off, l_off, o_off, q_off, bytes;
};

GqaLayout gqa_layout(int batch, int heads, int cap) {
    GqaLayout g;
    g.splits = (cap + la::kGqaChunk - 1) / la::kGqaChunk;
    const size_t n = (size_t)batch * heads * g.splits;
    auto up16 = [](size_t x) { return (x + 15) / 16 * 16; };
    g.m_off = 0;
    g.l_off = up16(n * 4);
    g.o_off = g.l_off + up16(n * 4);
    g.q_off = g.o_off + n * la::kGqaDim * 4;                           // rotated queries
    g.bytes = g.q_off + (size_t)batch * heads * la::kGqaDim * 4;
    return g;
}

template <typename T>
la_status run_gqa_decode(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                         const int *pos, int batch, int heads, int kv_heads, int cap, int rot, double base,
                         float scale, void *o, void *workspace, cudaStream_t stream) {
    const GqaLayout g = gqa_layout(batch, heads, cap);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *pm = reinterpret_cast<float *>(ws + g.m_off), *pl = reinterpret_cast<float *>(ws + g.l_off);
    float *po = reinterpret_cast<float *>(ws + g.o_off), *qr = reinterpret_cast<float *>(ws + g.q_off);
    la::gqa_append_kernel<T><<<dim3(batch, kv_heads), la::kGqaDim, 0, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k_new), static_cast<const T *>(v_new),
        static_cast<T *>(k_cache), static_cast<T *>(v_cache), pos, heads, kv_heads, cap, rot, base, scale, qr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gqa append launch");
    const bool bf16 = sizeof(T) == 2;
    if (bf16) {
        // bf16 cache: the chunks' partial softmax on the tensor cores
        CUtensorMap tk, tv;
        const long long bkv = (long long)batch * kv_heads;
        if (!la::gqp_make_map(&tk, k_cache, cap, cap, bkv, &g_last_error) ||
            !la::gqp_make_map(&tv, v_cache, cap, cap, bkv, &g_last_error))
            return LA_ERR_CUDA;
        e = cudaFuncSetAttribute(la::gqd::gqd_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)la::gqd::kSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gqd_partial)");
        la::gqd::gqd_partial_kernel<<<dim3(g.splits, kv_heads, batch), la::gqd::kThreads, la::gqd::kSmemBytes,
                                      stream>>>(tk, tv, qr, pos, heads, kv_heads, cap, g.splits, pm, pl, po);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "gqd partial launch");
        la::gqa_combine_kernel<T><<<(unsigned)((size_t)batch * heads), la::kGqaDim, 0, stream>>>(
            pm, pl, po, g.splits, static_cast<T *>(o));
        e = cudaGetLastError();
        return e == cudaSuccess ? ok() : cuda_fail(e, "gqa combine launch");
    }
    // f32 cache: CUDA cores. The caches as 2-D tensors [batch*kv_heads*cap][dim], 128-byte
    // swizzled boxes of one tile of positions
    const cuuint64_t rows = (cuuint64_t)batch * kv_heads * cap;
    CUtensorMap mk, mv;
    {
        auto fn = la::tc::encode_fn(&g_last_error);
        if (!fn) return LA_ERR_CUDA;
        const cuuint64_t dims[2] = {(cuuint64_t)la::kGqaDim, rows};
        const cuuint64_t strides[1] = {(cuuint64_t)la::kGqaDim * sizeof(T)};
        const cuuint32_t box[2] = {la::kGqaBoxRowBytes / (cuuint32_t)sizeof(T),
                                   (cuuint32_t)(la::kGqaTileBytes / (la::kGqaDim * sizeof(T)))};
        const cuuint32_t estr[2] = {1, 1};
        for (int i = 0; i < 2; ++i) {
            CUresult r = fn(i == 0 ? &mk : &mv, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                            2, i == 0 ? k_cache : v_cache, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS) {
                g_last_error = "cuTensorMapEncodeTiled failed for a cache (CUresult " + std::to_string((int)r) + ")";
                return LA_ERR_CUDA;
            }
        }
    }
    e = cudaFuncSetAttribute(la::gqa_partial_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)la::kGqaSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gqa_partial)");
    la::gqa_partial_kernel<T><<<dim3(g.splits, kv_heads, batch), la::kGqaThreads, la::kGqaSmemBytes, stream>>>(
        mk, mv, qr, pos, heads, kv_heads, cap, g.splits, pm, pl, po);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gqa partial launch");
    la::gqa_combine_kernel<T><<<(unsigned)((size_t)batch * heads), la::kGqaDim, 0, stream>>>(pm, pl, po, g.splits,
                                                                                         static_cast<T *>(o));
    e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "gqa combine launch");
}

// One launch of the CUDA-core kernel as a pass of the backward computation.
template <typename T, int D>
la_status launch_simt_pass(const void *q, const void *k, const void *v, const float *slopes, int batch,
                           int heads, int seq, int block, const float *state_in, void *o, float *state_out,
                           la::SimtPass pass, cudaStream_t stream) {
    auto kern = la::prefill_simt_kernel<T, D, true>;
    const size_t smem = la::simt_smem_bytes<D>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill_simt pass)");
    dim3 grid((unsigned)((size_t)batch * heads * (D / la::kSimtCols)));
    kern<<<grid, la::kSimtThreads, smem, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), slopes, heads, seq,
        block, state_in, static_cast<T *>(o), state_out, la::Snapshots{nullptr, 0, 0}, pass);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefill_simt pass launch");
    return ok();
}

struct BackwardArgs {
    const void *q, *k, *v, *d_o;
    la_dtype dtype;
    const float *slopes;
    int batch, heads, seq, dim, block;
    const float *state_in, *d_state_out;
    void *dq, *dk, *dv;
    float *d_state_in;
    void *workspace;
    size_t workspace_bytes;
};

// Scratch of lightning_prefill_backward_noalloc: a fixed device array, so that
// entry point needs no workspace from the caller and allocates nothing. 4 MiB
// hold the three passes' range-guard records for 29127 (batch, head) pairs.
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address, looked up once per device with that device current.
// In host code `g_noalloc_scratch` names a host-side stand-in, not the device
// memory, so a kernel must be given this address instead.
la_status noalloc_scratch(void **out) {
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(LA_ERR_UNSUPPORTED, "device ordinal %d above 63", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        addr[dev] = p;
    }
    *out = addr[dev];
    return LA_OK;
}

// Which kernels a backward request runs (LA_VARIANT_SIMT or _TCGEN05_PAIR), or -1.
int choose_backward_variant(la_dtype dtype, int dim, int block, int requested) {
    const bool pair_ok = la::pair_supports(dtype == LA_DTYPE_BF16, dim, block);
    switch (requested) {
        case LA_VARIANT_AUTO: return pair_ok ? LA_VARIANT_TCGEN05_PAIR : LA_VARIANT_SIMT;
        case LA_VARIANT_SIMT: return LA_VARIANT_SIMT;
        case LA_VARIANT_TCGEN05_PAIR: return pair_ok ? LA_VARIANT_TCGEN05_PAIR : -1;
        default: return -1;
    }
}

// Workspace a backward request needs: the range guard's records of the three
// tensor-core passes (dV, dK, dQ, one region each); none on CUDA cores.
size_t backward_workspace_bytes(la_dtype dtype, int batch, int heads, int seq, int dim, int variant) {
    (void)dtype; (void)seq; (void)dim;
    return variant == LA_VARIANT_TCGEN05_PAIR ? 3 * la::pair_workspace_bytes((long long)batch * heads) : 0;
}

la_status check_backward_pointers(const BackwardArgs &a) {
    const size_t eb = elem_bytes(a.dtype);
    const size_t n_tok = (size_t)a.batch * a.heads * a.seq * a.dim;
    const size_t n_state = (size_t)a.batch * a.heads * a.dim * a.dim;
    if (a.seq > 0 && (!a.q || !a.k || !a.v || !a.d_o || !a.dq || !a.dk || !a.dv))
        return fail(LA_ERR_INVALID_ARG, "q, k, v, d_o, dq, dk and dv must be non-NULL when seq > 0");
    if (!a.slopes) return fail(LA_ERR_INVALID_ARG, "slopes must be non-NULL");
    const void *ptrs[] = {a.q, a.k, a.v, a.d_o, a.slopes, a.state_in, a.d_state_out, a.dq, a.dk, a.dv,
                          a.d_state_in};
    const char *names[] = {"q", "k", "v", "d_o", "slopes", "state_in", "d_state_out", "dq", "dk", "dv",
                           "d_state_in"};
    for (int i = 0; i < 11; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(LA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    const size_t tok = a.seq > 0 ? n_tok * eb : 0;
    const Range in[] = {range_of(a.q, tok), range_of(a.k, tok), range_of(a.v, tok), range_of(a.d_o, tok),
                        range_of(a.slopes, sizeof(float) * a.heads),
                        range_of(a.state_in, a.state_in ? n_state * 4 : 0),
                        range_of(a.d_state_out, a.d_state_out ? n_state * 4 : 0)};
    const Range out[] = {range_of(a.dq, tok), range_of(a.dk, tok), range_of(a.dv, tok),
                         range_of(a.d_state_in, a.d_state_in ? n_state * 4 : 0)};
    for (int i = 0; i < 4; ++i) {
        for (const Range &r : in)
            if (overlaps(out[i], r)) return fail(LA_ERR_INVALID_ARG, "a gradient output overlaps an input");
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(out[i], out[j])) return fail(LA_ERR_INVALID_ARG, "two gradient outputs overlap");
    }
    return LA_OK;
}

la_status check_backward_workspace(const BackwardArgs &a, size_t need) {
    if (need == 0 || a.seq == 0 || a.batch == 0) return LA_OK;
    if (!a.workspace || a.workspace_bytes < need)
        return fail(LA_ERR_INVALID_ARG, "the tensor-core backward needs %zu bytes of workspace (got %zu)", need,
                    a.workspace ? a.workspace_bytes : (size_t)0);
    if (!aligned16(a.workspace)) return fail(LA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    const size_t eb = elem_bytes(a.dtype);
    const size_t n_tok = (size_t)a.batch * a.heads * a.seq * a.dim;
    const size_t n_state = (size_t)a.batch * a.heads * a.dim * a.dim;
    const Range rw = range_of(a.workspace, need);
    const Range others[] = {range_of(a.q, n_tok * eb), range_of(a.k, n_tok * eb), range_of(a.v, n_tok * eb),
                            range_of(a.d_o, n_tok * eb), range_of(a.dq, n_tok * eb), range_of(a.dk, n_tok * eb),
                            range_of(a.dv, n_tok * eb), range_of(a.slopes, sizeof(float) * a.heads),
                            range_of(a.state_in, a.state_in ? n_state * 4 : 0),
                            range_of(a.d_state_out, a.d_state_out ? n_state * 4 : 0),
                            range_of(a.d_state_in, a.d_state_in ? n_state * 4 : 0)};
    for (const Range &r : others)
        if (overlaps(rw, r)) return fail(LA_ERR_INVALID_ARG, "workspace overlaps an input or an output");
    return LA_OK;
}

// The tensor-core backward: the three passes on the CTA-pair kernel. dQ runs
// causal on (dO, V, K) with the carried state S_in^T; dV and dK run
// anti-causal (blocks from last to first, state anchored at each block's last
// token) on (K, Q, dO) with carried state dS_out, whose final state is dS_in,
// and on (V, dO, Q) with dS_out^T.
// Two auxiliary streams per device, created on first use and kept for the process:
// the backward passes run side by side on them.
cudaError_t aux_streams(cudaStream_t (&out)[2]) {
    static std::mutex mu;
    static cudaStream_t streams[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 2; ++i)
        if (!streams[dev][i]) {
            e = cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking);
            if (e != cudaSuccess) return e;
        }
    out[0] = streams[dev][0];
    out[1] = streams[dev][1];
    return cudaSuccess;
}

// The three passes read the same inputs and write disjoint outputs, and each launch fills
// only 2 SMs per (batch, head): dV and dK go to two auxiliary streams forked from and joined
// back into `stream` with events, so that a pass's CTA pairs start on the SMs the others
// leave free. Enqueue order on `stream` is kept (the fork waits for everything before it,
// and everything after waits for the join), and the pattern can be captured into a graph.
la_status run_backward_pair(const BackwardArgs &a, cudaStream_t stream) {
    const la::Snapshots none{nullptr, 0, 0};
    la::rg::RangeRec *rec = static_cast<la::rg::RangeRec *>(a.workspace);
    const size_t per_pass = (size_t)a.batch * a.heads;
    cudaStream_t aux[2];
    cudaError_t e = aux_streams(aux);
    if (e != cudaSuccess) return cuda_fail(e, "creating the backward's auxiliary streams");
    cudaEvent_t fork, join[2];
    e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
    for (int i = 0; i < 2; ++i)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join[i], cudaEventDisableTiming);
    la_status st = LA_OK;
    if (e != cudaSuccess) st = cuda_fail(e, "cudaEventCreate");
    if (st == LA_OK) {
        e = cudaEventRecord(fork, stream);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(aux[i], fork, 0);
        if (e != cudaSuccess) st = cuda_fail(e, "forking the backward passes");
    }
    if (st == LA_OK)
        st = la::launch_pair(a.k, a.q, a.d_o, a.slopes, a.batch, a.heads, a.seq, a.d_state_out, a.dv, a.d_state_in,
                             none, la::pair::PairPass{0, 1}, rec, aux[0], &g_last_error);
    if (st == LA_OK)
        st = la::launch_pair(a.v, a.d_o, a.q, a.slopes, a.batch, a.heads, a.seq, a.d_state_out, a.dk, nullptr,
                             none, la::pair::PairPass{1, 1}, rec + per_pass, aux[1], &g_last_error);
    if (st == LA_OK)
        st = la::launch_pair(a.d_o, a.v, a.k, a.slopes, a.batch, a.heads, a.seq, a.state_in, a.dq, nullptr, none,
                             la::pair::PairPass{1, 0}, rec + 2 * per_pass, stream, &g_last_error);
    // join even after a failed launch, so that `stream` never runs ahead of work already enqueued
    for (int i = 0; i < 2; ++i) {
        cudaError_t r = cudaEventRecord(join[i], aux[i]);
        if (r == cudaSuccess) r = cudaStreamWaitEvent(stream, join[i], 0);
        if (r != cudaSuccess && st == LA_OK) st = cuda_fail(r, "joining the backward passes");
    }
    cudaEventDestroy(fork);
    for (int i = 0; i < 2; ++i) cudaEventDestroy(join[i]);
    return st;
}

// The gradients as three passes of the block recurrence (see lightning.h):
//   dQ: forward in time, (q, k, v) <- (dO, V, K), carried state S_in^T;
//   dV: backward in time, (q, k, v) <- (K, Q, dO), carried state dS_out seen
//       from the last token on, final state times e^{-s} = dS_in;
//   dK: backward in time, (q, k, v) <- (V, dO, Q), carried state dS_out^T.
template <typename T, int D>
la_status run_backward_typed(const BackwardArgs &a, cudaStream_t stream) {
    la_status st = launch_simt_pass<T, D>(a.d_o, a.v, a.k, a.slopes, a.batch, a.heads, a.seq, a.block, a.state_in,
                                          a.dq, nullptr, la::SimtPass{0, 1, 0, 0}, stream);
    if (st != LA_OK) return st;
    st = launch_simt_pass<T, D>(a.k, a.q, a.d_o, a.slopes, a.batch, a.heads, a.seq, a.block, a.d_state_out,
                                a.dv, a.d_state_in, la::SimtPass{1, 0, 1, 1}, stream);
    if (st != LA_OK) return st;
    return launch_simt_pass<T, D>(a.v, a.d_o, a.q, a.slopes, a.batch, a.heads, a.seq, a.block, a.d_state_out,
                                  a.dk, nullptr, la::SimtPass{1, 1, 1, 0}, stream);
}

la_status run_backward(const BackwardArgs &a, cudaStream_t stream, int variant) {
    if (a.batch == 0 || (a.seq == 0 && !a.d_state_in)) return ok();
    if (const la_status early = earlier_failure()) return early;
    if (a.seq == 0) {
        // no token: the state passes through, and so does its gradient
        const size_t n = (size_t)a.batch * a.heads * a.dim * a.dim;
        la::state_passthrough_kernel<<<(unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0,
                                       stream>>>(a.d_state_out, a.d_state_in, n);
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? ok() : cuda_fail(e, "state gradient passthrough launch");
    }
    if (variant == LA_VARIANT_TCGEN05_PAIR) return run_backward_pair(a, stream);
    if (a.dtype == LA_DTYPE_BF16)
        return a.dim == 64 ? run_backward_typed<__nv_bfloat16, 64>(a, stream)
                           : run_backward_typed<__nv_bfloat16, 128>(a, stream);
    return a.dim == 64 ? run_backward_typed<float, 64>(a, stream) : run_backward_typed<float, 128>(a, stream);
}

la_status run_prefill(const PrefillArgs &a, cudaStream_t stream, int variant) {
    if (a.batch == 0 || (a.seq == 0 && !a.state_out)) return ok();
    if (const la_status early = earlier_failure()) return early;
    if (a.seq == 0) {
        const size_t n = (size_t)a.batch * a.heads * a.dim * a.dim;
        la::state_passthrough_kernel<<<(unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0,
                                       stream>>>(a.state_in, a.state_out, n);
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? ok() : cuda_fail(e, "state passthrough launch");
    }
    if (variant == LA_VARIANT_TCGEN05_PAIR)
        return la::launch_pair(a.q, a.k, a.v, a.slopes, a.batch, a.heads, a.seq, a.state_in, a.o, a.state_out,
                               a.sn, la::pair::PairPass{0, 0}, static_cast<la::rg::RangeRec *>(a.workspace), stream,
                               &g_last_error);
    if (variant == LA_VARIANT_TCGEN05) return la::launch_tc(a.q, a.k, a.v, a.slopes, a.batch, a.heads,
                                                           a.seq, a.block, a.state_in, a.o, a.state_out,
                                                           a.sn, static_cast<la::rg::RangeRec *>(a.workspace),
                                                           stream, &g_last_error);
    if (a.dtype == LA_DTYPE_BF16)
        return a.dim == 64 ? launch_simt<__nv_bfloat16, 64>(a, stream)
                           : launch_simt<__nv_bfloat16, 128>(a, stream);
    return a.dim == 64 ? launch_simt<float, 64>(a, stream) : launch_simt<float, 128>(a, stream);
}

template <typename T, int D>
la_status launch_decode(const void *q, const void *k, const void *v, const float *slopes, int batch,
                        int heads, float *state, void *o, cudaStream_t stream) {
    la::decode_kernel<T, D><<<(unsigned)((size_t)batch * heads), la::kDecodeThreads, 0, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), slopes, heads,
        state, static_cast<T *>(o));
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "decode launch");
}

}  // namespace

extern "C" {

int lightning_abi_version(void) { return 2; }

}  // extern "C"

namespace {

// Shared path of every prefill entry point: shape, variant, pointers, launch.
la_status prefill_entry(const PrefillArgs &a, void *stream, int variant, bool with_snapshots) {
    const la_dtype dtype = a.dtype;
    const int dim = a.dim, block = a.block;
    la_status st = check_prefill_shape(dtype, a.batch, a.heads, a.seq, dim, block);
    if (st != LA_OK) return st;
    const int chosen = choose_variant(dtype, dim, block, variant);
    if (chosen < 0) {
        if (variant < LA_VARIANT_AUTO || variant > LA_VARIANT_TCGEN05_PAIR)
            return fail(LA_ERR_INVALID_ARG, "unknown variant %d", variant);
        return fail(LA_ERR_UNSUPPORTED,
                    "the tcgen05 kernels need bf16 and dim 128, with block 128 or 256 (single CTA) or block 256 "
                    "(CTA pair) (got dtype %d, dim %d, block %d)",
                    (int)dtype, dim, block);
    }
    st = check_prefill_pointers(a);
    if (st != LA_OK) return st;
    if (with_snapshots) {
        st = check_snapshots(a);
        if (st != LA_OK) return st;
    }
    st = check_prefill_workspace(a, chosen);
    if (st != LA_OK) return st;
    return run_prefill(a, static_cast<cudaStream_t>(stream), chosen);
}

}  // namespace

extern "C" {

la_status lightning_prefill_ex(const void *q, const void *k, const void *v, la_dtype dtype,
                               const float *slopes, int batch, int heads, int seq, int dim, int block,
                               const float *state_in, void *o, float *state_out, void *workspace,
                               size_t workspace_bytes, void *stream, int variant) {
    const PrefillArgs a{q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, o, state_out,
                        la::Snapshots{nullptr, 0, 0}, workspace, workspace_bytes};
    return prefill_entry(a, stream, variant, false);
}

la_status lightning_prefill_backward(const void *q, const void *k, const void *v, const void *d_o,
                                     la_dtype dtype, const float *slopes, int batch, int heads, int seq,
                                     int dim, int block, const float *state_in, const float *d_state_out,
                                     void *dq, void *dk, void *dv, float *d_state_in, void *workspace,
                                     size_t workspace_bytes, void *stream, int variant) {
    la_status st = check_prefill_shape(dtype, batch, heads, seq, dim, block);
    if (st != LA_OK) return st;
    const int chosen = choose_backward_variant(dtype, dim, block, variant);
    if (chosen < 0) {
        if (variant < LA_VARIANT_AUTO || variant > LA_VARIANT_TCGEN05_PAIR || variant == LA_VARIANT_TCGEN05)
            return fail(LA_ERR_INVALID_ARG, "variant %d is not a backward variant (AUTO, SIMT or TCGEN05_PAIR)",
                        variant);
        return fail(LA_ERR_UNSUPPORTED, "the tensor-core backward needs bf16, dim 128 and block 256");
    }
    const BackwardArgs a{q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block, state_in, d_state_out,
                         dq, dk, dv, d_state_in, workspace, workspace_bytes};
    st = check_backward_pointers(a);
    if (st != LA_OK) return st;
    st = check_backward_workspace(a, backward_workspace_bytes(dtype, batch, heads, seq, dim, chosen));
    if (st != LA_OK) return st;
    return run_backward(a, static_cast<cudaStream_t>(stream), chosen);
}

la_status lightning_prefill_backward_noalloc(const void *q, const void *k, const void *v, const void *d_o,
                                             la_dtype dtype, const float *slopes, int batch, int heads, int seq,
                                             int dim, int block, const float *state_in, const float *d_state_out,
                                             void *dq, void *dk, void *dv, float *d_state_in, void *stream,
                                             int variant) {
    // the same argument checks, in the same order, as lightning_prefill_backward
    la_status st = check_prefill_shape(dtype, batch, heads, seq, dim, block);
    if (st != LA_OK) return st;
    const int chosen = choose_backward_variant(dtype, dim, block, variant);
    if (chosen < 0)  // its own message for an unknown or unsupported variant
        return lightning_prefill_backward(q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block, state_in,
                                          d_state_out, dq, dk, dv, d_state_in, nullptr, 0, stream, variant);
    const BackwardArgs a{q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block, state_in, d_state_out,
                         dq, dk, dv, d_state_in, nullptr, 0};
    st = check_backward_pointers(a);
    if (st != LA_OK) return st;
    const size_t need = backward_workspace_bytes(dtype, batch, heads, seq, dim, chosen);
    if (need > kNoAllocScratchBytes)
        return fail(LA_ERR_UNSUPPORTED, "the request needs %zu bytes of scratch; the built-in scratch holds %zu",
                    need, kNoAllocScratchBytes);
    void *scratch = nullptr;
    if (need > 0 && batch > 0 && seq > 0) {
        st = noalloc_scratch(&scratch);
        if (st != LA_OK) return st;
    }
    return lightning_prefill_backward(q, k, v, d_o, dtype, slopes, batch, heads, seq, dim, block, state_in,
                                      d_state_out, dq, dk, dv, d_state_in, scratch, need, stream, variant);
}

size_t lightning_prefill_backward_noalloc_capacity(void) { return kNoAllocScratchBytes; }

size_t lightning_prefill_backward_workspace_size(la_dtype dtype, int batch, int heads, int seq, int dim,
                                                 int block, int variant) {
    if (check_prefill_shape(dtype, batch, heads, seq, dim, block) != LA_OK) return 0;
    const int chosen = choose_backward_variant(dtype, dim, block, variant);
    return chosen < 0 ? 0 : backward_workspace_bytes(dtype, batch, heads, seq, dim, chosen);
}

la_status lightning_prefill_norm_gate(const void *q, const void *k, const void *v, la_dtype dtype,
                                      const float *slopes, int batch, int heads, int seq, int dim, int block,
                                      const float *state_in, const void *gate, const float *gamma, float eps,
                                      void *y, float *state_out, void *workspace, size_t workspace_bytes,
                                      void *stream) {
    la_status st = check_prefill_shape(dtype, batch, heads, seq, dim, block);
    if (st != LA_OK) return st;
    if (!la::pair_supports(dtype == LA_DTYPE_BF16, dim, block))
        return fail(LA_ERR_UNSUPPORTED,
                    "the fused normalisation runs on the CTA-pair kernel: bf16, dim 128, block 256 (got dtype %d, "
                    "dim %d, block %d)",
                    (int)dtype, dim, block);
    if (!(eps >= 0.f) || eps > 3.0e38f) return fail(LA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const PrefillArgs a{q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, y, state_out,
                        la::Snapshots{nullptr, 0, 0}, workspace, workspace_bytes};
    st = check_prefill_pointers(a);
    if (st != LA_OK) return st;
    const size_t n_tok = (size_t)batch * heads * seq * dim;
    if (n_tok > 0) {
        if (!gate || !gamma) return fail(LA_ERR_INVALID_ARG, "gate and gamma must be non-NULL when seq > 0");
        if (!aligned16(gate) || !aligned16(gamma))
            return fail(LA_ERR_INVALID_ARG, "gate and gamma must be 16-byte aligned");
        const Range ry = range_of(y, n_tok * 2);
        if (overlaps(ry, range_of(gate, n_tok * 2)) || overlaps(ry, range_of(gamma, sizeof(float) * heads * dim)))
            return fail(LA_ERR_INVALID_ARG, "y overlaps gate or gamma");
        if (state_out) {
            const Range rs = range_of(state_out, (size_t)batch * heads * dim * dim * 4);
            if (overlaps(rs, range_of(gate, n_tok * 2)) || overlaps(rs, range_of(gamma, sizeof(float) * heads * dim)))
                return fail(LA_ERR_INVALID_ARG, "state_out overlaps gate or gamma");
        }
        st = check_prefill_workspace(a, LA_VARIANT_TCGEN05_PAIR);
        if (st != LA_OK) return st;
        const Range rw = range_of(workspace, prefill_workspace_bytes(batch, heads, LA_VARIANT_TCGEN05_PAIR));
        if (overlaps(rw, range_of(gate, n_tok * 2)) || overlaps(rw, range_of(gamma, sizeof(float) * heads * dim)))
            return fail(LA_ERR_INVALID_ARG, "workspace overlaps gate or gamma");
    }
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (batch == 0 || seq == 0) return run_prefill(a, cs, LA_VARIANT_TCGEN05_PAIR);
    if (const la_status early = earlier_failure()) return early;
    const la::pair::PairNormGate ng{static_cast<const __nv_bfloat16 *>(gate), gamma, eps};
    return la::launch_pair(q, k, v, slopes, batch, heads, seq, state_in, y, state_out, a.sn, la::pair::PairPass{0, 0},
                           static_cast<la::rg::RangeRec *>(workspace), cs, &g_last_error, &ng);
}

la_status lightning_norm_gate(const void *o, const void *gate, la_dtype dtype, const float *gamma, float eps,
                              int batch, int heads, int seq, int dim, int per_head, void *y, void *stream) {
    if (dtype != LA_DTYPE_F32 && dtype != LA_DTYPE_BF16)
        return fail(LA_ERR_INVALID_ARG, "dtype %d is neither LA_DTYPE_F32 nor LA_DTYPE_BF16", (int)dtype);
    if (batch < 0 || heads < 1 || seq < 0)
        return fail(LA_ERR_INVALID_ARG, "need batch >= 0, heads >= 1, seq >= 0 (got %d, %d, %d)", batch, heads, seq);
    if (!(eps >= 0.f) || eps > 3.0e38f) return fail(LA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (dim != 64 && dim != 128) return fail(LA_ERR_UNSUPPORTED, "dim %d unsupported (64 or 128)", dim);
    const size_t eb = elem_bytes(dtype);
    const long long max_ch = (long long)la::kNgGroup * la::kNgMaxChunks * (long long)(16 / eb);
    if ((long long)heads * dim > max_ch)
        return fail(LA_ERR_UNSUPPORTED, "heads*dim %lld exceeds %lld channels per token",
                    (long long)heads * dim, max_ch);
    const long long tokens = (long long)batch * seq;
    if (tokens == 0) return ok();
    if (!o || !gate || !gamma || !y) return fail(LA_ERR_INVALID_ARG, "o, gate, gamma and y must be non-NULL");
    const void *ptrs[] = {o, gate, gamma, y};
    const char *names[] = {"o", "gate", "gamma", "y"};
    for (int i = 0; i < 4; ++i)
        if (!aligned16(ptrs[i])) return fail(LA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    const size_t bytes = (size_t)tokens * heads * dim * eb;
    const Range ry = range_of(y, bytes);
    if (overlaps(ry, range_of(o, bytes)) || overlaps(ry, range_of(gate, bytes)) ||
        overlaps(ry, range_of(gamma, sizeof(float) * heads * dim)))
        return fail(LA_ERR_INVALID_ARG, "y overlaps o, gate or gamma");
    // chunks of 16 bytes per thread, and resident CTAs on every SM, each walking the tokens
    const long long chunks_per_thread = ((long long)heads * dim * (long long)eb / 16 + la::kNgGroup - 1) / la::kNgGroup;
    const int U = chunks_per_thread <= 1 ? 1 : chunks_per_thread <= 2 ? 2 : chunks_per_thread <= 4 ? 4 : 8;
    if (const la_status early = earlier_failure()) return early;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const NgArgs args{o, gate, gamma, eps, batch, heads, seq, dim, per_head ? 1 : 0, y, tokens, st};
    la_status rs;
    if (dtype == LA_DTYPE_BF16)
        rs = U == 1 ? launch_norm_gate<__nv_bfloat16, 1>(args) : U == 2 ? launch_norm_gate<__nv_bfloat16, 2>(args)
           : U == 4 ? launch_norm_gate<__nv_bfloat16, 4>(args) : launch_norm_gate<__nv_bfloat16, 8>(args);
    else
        rs = U == 1 ? launch_norm_gate<float, 1>(args) : U == 2 ? launch_norm_gate<float, 2>(args)
           : U == 4 ? launch_norm_gate<float, 4>(args) : launch_norm_gate<float, 8>(args);
    return rs;
}


size_t lightning_gqa_decode_workspace_size(int batch, int heads, int cap) {
    if (batch < 0 || heads < 1 || cap < 1) return 0;
    return gqa_layout(batch, heads, cap).bytes;
}

la_status lightning_gqa_decode(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                               la_dtype dtype, const int *pos, int batch, int heads, int kv_heads, int dim, int cap,
                               int rot, double rope_base, float scale, void *o, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (dtype != LA_DTYPE_F32 && dtype != LA_DTYPE_BF16)
        return fail(LA_ERR_INVALID_ARG, "dtype %d is neither LA_DTYPE_F32 nor LA_DTYPE_BF16", (int)dtype);
    if (batch < 0 || heads < 1 || kv_heads < 1 || cap < 1 || heads % kv_heads != 0)
        return fail(LA_ERR_INVALID_ARG, "need batch >= 0, cap >= 1 and kv_heads dividing heads (got %d, %d, %d, %d)",
                    batch, cap, heads, kv_heads);
    if (dim != la::kGqaDim) return fail(LA_ERR_UNSUPPORTED, "dim %d unsupported (128)", dim);
    // bf16: the group's heads are rows handled by one 32-lane softmax warp; float32: the
    // CUDA-core kernel keeps kGqaMaxGroup heads in registers
    const int max_group = dtype == LA_DTYPE_BF16 ? 32 : la::kGqaMaxGroup;
    if (heads / kv_heads > max_group)
        return fail(LA_ERR_UNSUPPORTED, "at most %d query heads per KV head for this dtype (got %d)", max_group,
                    heads / kv_heads);
    if (rot < 0 || rot > dim || (rot & 1)) return fail(LA_ERR_INVALID_ARG, "rot must be even, 0 <= rot <= dim");
    if (!(rope_base > 0.0) || rope_base > 1e300) return fail(LA_ERR_INVALID_ARG, "rope_base must be finite and > 0");
    if (!(scale == scale) || scale > 3e38f || scale < -3e38f) return fail(LA_ERR_INVALID_ARG, "scale must be finite");
    if (batch == 0) return ok();
    const GqaLayout g = gqa_layout(batch, heads, cap);
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o)
        return fail(LA_ERR_INVALID_ARG, "q, k_new, v_new, the caches, pos and o must be non-NULL");
    if (!workspace || workspace_bytes < g.bytes)
        return fail(LA_ERR_INVALID_ARG, "workspace needs %zu bytes (got %zu)", g.bytes,
                    workspace ? workspace_bytes : (size_t)0);
    const void *ptrs[] = {q, k_new, v_new, k_cache, v_cache, pos, o, workspace};
    const char *names[] = {"q", "k_new", "v_new", "k_cache", "v_cache", "pos", "o", "workspace"};
    for (int i = 0; i < 8; ++i)
        if (!aligned16(ptrs[i])) return fail(LA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    const size_t eb = elem_bytes(dtype);
    const size_t nq = (size_t)batch * heads * dim * eb, nkv = (size_t)batch * kv_heads * dim * eb;
    const size_t ncache = (size_t)batch * kv_heads * cap * dim * eb;
    const Range rq = range_of(q, nq), rkn = range_of(k_new, nkv), rvn = range_of(v_new, nkv);
    const Range rkc = range_of(k_cache, ncache), rvc = range_of(v_cache, ncache), rp = range_of(pos, 4 * batch);
    const Range ro = range_of(o, nq), rw = range_of(workspace, g.bytes);
    const Range all[] = {rq, rkn, rvn, rkc, rvc, rp, ro, rw};
    const int written[] = {3, 4, 6, 7};  // the caches, o and the workspace
    for (int wi : written)
        for (int j = 0; j < 8; ++j)
            if (j != wi && overlaps(all[wi], all[j]))
                return fail(LA_ERR_INVALID_ARG, "%s overlaps %s", names[wi], names[j]);
    if (const la_status early = earlier_failure()) return early;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dtype == LA_DTYPE_BF16)
        return run_gqa_decode<__nv_bfloat16>(q, k_new, v_new, k_cache, v_cache, pos, batch, heads, kv_heads, cap, rot,
                                             rope_base, scale, o, workspace, st);
    return run_gqa_decode<float>(q, k_new, v_new, k_cache, v_cache, pos, batch, heads, kv_heads, cap, rot, rope_base,
                                 scale, o, workspace, st);
}

size_t lightning_gqa_prefill_workspace_size(la_dtype dtype, int batch, int heads, int seq, int dim) {
    if ((dtype != LA_DTYPE_F32 && dtype != LA_DTYPE_BF16) || batch < 0 || heads < 1 || seq < 0 || dim != la::gqp::kDim)
        return 0;
    return (size_t)batch * heads * seq * dim * elem_bytes(dtype);  // the rotated queries
}

la_status lightning_gqa_prefill(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                                la_dtype dtype, const int *start, int batch, int heads, int kv_heads, int seq, int dim,
                                int cap, int rot, double rope_base, float scale, void *o, void *workspace,
                                size_t workspace_bytes, void *stream) {
    if (dtype != LA_DTYPE_F32 && dtype != LA_DTYPE_BF16)
        return fail(LA_ERR_INVALID_ARG, "dtype %d is neither LA_DTYPE_F32 nor LA_DTYPE_BF16", (int)dtype);
    if (batch < 0 || seq < 0 || heads < 1 || kv_heads < 1 || cap < 1 || heads % kv_heads != 0)
        return fail(LA_ERR_INVALID_ARG,
                    "need batch, seq >= 0, cap >= 1 and kv_heads dividing heads (got %d, %d, %d, %d, %d)", batch, seq,
                    cap, heads, kv_heads);
    if (seq > cap) return fail(LA_ERR_INVALID_ARG, "seq %d exceeds cap %d", seq, cap);
    if (dim != la::gqp::kDim) return fail(LA_ERR_UNSUPPORTED, "dim %d unsupported (128)", dim);
    if (rot < 0 || rot > dim || (rot & 3)) return fail(LA_ERR_INVALID_ARG, "rot must be a multiple of 4, 0 <= rot <= dim");
    if (!(rope_base > 0.0) || rope_base > 1e300) return fail(LA_ERR_INVALID_ARG, "rope_base must be finite and > 0");
    if (!(scale > 0.f) || scale > 3e38f) return fail(LA_ERR_INVALID_ARG, "scale must be finite and > 0");
    if (batch > 65535) return fail(LA_ERR_UNSUPPORTED, "batch %d above 65535", batch);
    if (batch == 0 || seq == 0) return ok();
    const long long ctas = (long long)batch * heads * ((seq + la::gqp::kQRows - 1) / la::gqp::kQRows);
    if (ctas > 0x7fffffffLL) return fail(LA_ERR_UNSUPPORTED, "problem too large for one launch");
    const size_t need = lightning_gqa_prefill_workspace_size(dtype, batch, heads, seq, dim);
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !o || !start)
        return fail(LA_ERR_INVALID_ARG, "q, k_new, v_new, the caches, start and o must be non-NULL");
    if (!workspace || workspace_bytes < need)
        return fail(LA_ERR_INVALID_ARG, "workspace needs %zu bytes (got %zu)", need, workspace ? workspace_bytes : (size_t)0);
    const void *ptrs[] = {q, k_new, v_new, k_cache, v_cache, o, workspace, start};
    const char *names[] = {"q", "k_new", "v_new", "k_cache", "v_cache", "o", "workspace", "start"};
    for (int i = 0; i < 8; ++i)
        if (!aligned16(ptrs[i])) return fail(LA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    const size_t eb = elem_bytes(dtype);
    const size_t nq = (size_t)batch * heads * seq * dim * eb, nkv = (size_t)batch * kv_heads * seq * dim * eb;
    const size_t ncache = (size_t)batch * kv_heads * cap * dim * eb;
    const Range all[] = {range_of(q, nq), range_of(k_new, nkv), range_of(v_new, nkv), range_of(k_cache, ncache),
                         range_of(v_cache, ncache), range_of(o, nq), range_of(workspace, need),
                         range_of(start, sizeof(int) * batch)};
    const int written[] = {3, 4, 5, 6};  // the caches, o and the workspace
    for (int wi : written)
        for (int j = 0; j < 8; ++j)
            if (j != wi && overlaps(all[wi], all[j]))
                return fail(LA_ERR_INVALID_ARG, "%s overlaps %s", names[wi], names[j]);
    if (const la_status early = earlier_failure()) return early;
    if (dtype == LA_DTYPE_F32)
        return la::launch_gqa_prefill_f32(q, k_new, v_new, k_cache, v_cache, start, batch, heads, kv_heads, seq, cap,
                                          rot, rope_base, scale, o, workspace, static_cast<cudaStream_t>(stream),
                                          &g_last_error);
    return la::launch_gqa_prefill(q, k_new, v_new, k_cache, v_cache, start, batch, heads, kv_heads, seq, cap, rot,
                                  rope_base, scale, o, workspace, static_cast<cudaStream_t>(stream), &g_last_error);
}

int lightning_prefill_snapshot_count(int seq, int interval) {
    if (seq < 0 || interval < 1) return -1;
    return seq / interval;
}

la_status lightning_prefill_snapshots(const void *q, const void *k, const void *v, la_dtype dtype,
                                      const float *slopes, int batch, int heads, int seq, int dim, int block,
                                      const float *state_in, void *o, float *state_out, int interval,
                                      float *snapshots, void *workspace, size_t workspace_bytes, void *stream,
                                      int variant) {
    const int count = interval > 0 && seq >= 0 ? seq / interval : 0;
    const PrefillArgs a{q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, o, state_out,
                        la::Snapshots{count > 0 ? snapshots : nullptr, interval, count}, workspace, workspace_bytes};
    return prefill_entry(a, stream, variant, true);
}

la_status lightning_prefill(const void *q, const void *k, const void *v, la_dtype dtype,
                            const float *slopes, int batch, int heads, int seq, int dim, int block,
                            const float *state_in, void *o, float *state_out, void *workspace,
                            size_t workspace_bytes, void *stream) {
    return lightning_prefill_ex(q, k, v, dtype, slopes, batch, heads, seq, dim, block, state_in, o,
                                state_out, workspace, workspace_bytes, stream, LA_VARIANT_AUTO);
}

int lightning_prefill_selected_variant(la_dtype dtype, int batch, int heads, int seq, int dim, int block,
                                       int variant) {
    if (check_prefill_shape(dtype, batch, heads, seq, dim, block) != LA_OK) return -1;
    return choose_variant(dtype, dim, block, variant);
}

size_t lightning_prefill_workspace_size(int batch, int heads, int seq, int dim, int block) {
    if (check_prefill_shape(LA_DTYPE_BF16, batch, heads, seq, dim, block) != LA_OK) return 0;
    // the largest any kernel takes for these sizes (bf16 inputs)
    return prefill_workspace_bytes(batch, heads, choose_variant(LA_DTYPE_BF16, dim, block, LA_VARIANT_AUTO));
}

la_status lightning_decode(const void *q, const void *k, const void *v, la_dtype dtype, const float *slopes,
                           int batch, int heads, int dim, float *state, void *o, void *stream) {
    if (dtype != LA_DTYPE_F32 && dtype != LA_DTYPE_BF16)
        return fail(LA_ERR_INVALID_ARG, "dtype %d is neither LA_DTYPE_F32 nor LA_DTYPE_BF16", (int)dtype);
    if (batch < 0 || heads < 1)
        return fail(LA_ERR_INVALID_ARG, "need batch >= 0 and heads >= 1 (got %d, %d)", batch, heads);
    if (dim != 64 && dim != 128) return fail(LA_ERR_UNSUPPORTED, "dim %d unsupported (64 or 128)", dim);
    if ((long long)batch * heads > (1ll << 31) - 1) return fail(LA_ERR_UNSUPPORTED, "batch*heads too large");
    if (batch == 0) return ok();
    if (!q || !k || !v || !slopes || !state || !o)
        return fail(LA_ERR_INVALID_ARG, "q, k, v, slopes, state and o must be non-NULL");
    const void *ptrs[] = {q, k, v, slopes, state, o};
    const char *names[] = {"q", "k", "v", "slopes", "state", "o"};
    for (int i = 0; i < 6; ++i)
        if (!aligned16(ptrs[i])) return fail(LA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    const size_t eb = elem_bytes(dtype);
    const size_t n_tok = (size_t)batch * heads * dim;
    const Range ro = range_of(o, n_tok * eb), rs = range_of(state, n_tok * dim * 4);
    const Range rin[] = {range_of(q, n_tok * eb), range_of(k, n_tok * eb), range_of(v, n_tok * eb),
                         range_of(slopes, sizeof(float) * heads)};
    if (overlaps(ro, rs)) return fail(LA_ERR_INVALID_ARG, "o overlaps the state");
    for (const Range &r : rin) {
        if (overlaps(ro, r)) return fail(LA_ERR_INVALID_ARG, "o overlaps an input");
        if (overlaps(rs, r)) return fail(LA_ERR_INVALID_ARG, "state overlaps an input");
    }
    if (const la_status early = earlier_failure()) return early;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == LA_DTYPE_BF16)
        return dim == 64 ? launch_decode<__nv_bfloat16, 64>(q, k, v, slopes, batch, heads, state, o, s)
                         : launch_decode<__nv_bfloat16, 128>(q, k, v, slopes, batch, heads, state, o, s);
    return dim == 64 ? launch_decode<float, 64>(q, k, v, slopes, batch, heads, state, o, s)
                     : launch_decode<float, 128>(q, k, v, slopes, batch, heads, state, o, s);
}

la_status lightning_last_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    const la_status st = status_of_word(__atomic_exchange_n(&la::g_device_status, 0u, __ATOMIC_ACQ_REL));
    return st == LA_OK ? ok() : st;
}

la_status lightning_device_status(void *stream) { return lightning_last_device_status(stream); }

la_status lightning_selftest_wait_timeout(void *stream) {
    la::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ok() : cuda_fail(e, "self-test launch");
}

const char *lightning_status_string(int status) {
    switch (status) {
        case LA_OK: return "LA_OK: success";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: no kernel for this request";
        case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA runtime error";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT: a device-side wait gave up";
        default: return "unknown status";
    }
}

const char *lightning_last_error_message(void) { return g_last_error.c_str(); }

}  // extern "C"
