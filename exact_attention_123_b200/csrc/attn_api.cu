// attn_api.cu -- the libattn C ABI: argument validation, TMA tensor-map
// construction, the device status word, and dispatch to the sm_100a launchers.
// No entry point allocates memory or synchronises, except attn_status().
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "../../include/libattn.h"
#include "attn_launch.h"

namespace {

__device__ int g_attn_status = 0;

// Test hook kernel: the forward kernels' FMA-pipe exponential on pairs of inputs.
__global__ void ex2_poly_probe_kernel(const float2 *x, float2 *y, long long pairs) {
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < pairs;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float2 v = x[i];
        float a, b;
        attn::ex2_poly_x2(attn::f2_pack(v.x, v.y), a, b);
        y[i] = make_float2(a, b);
    }
}

constexpr int kMaxDevices = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::atomic<int> g_wait_limit_ms{4000};
std::atomic<int> g_skip_load{-1};
std::atomic<int> g_bad_tag{-1};
std::atomic<int> g_force_band{0};  // test hook: slices per band forced (0: automatic)

struct DeviceState {
    std::once_flag once;
    int supported = 0;  // 1 if sm_100
    int num_sms = 0;
    int *status = nullptr;
    cudaError_t err = cudaSuccess;
};
DeviceState g_dev[kMaxDevices];

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Per-device one-time setup: architecture check and the status word's address.
int device_state(DeviceState **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
    DeviceState &s = g_dev[dev];
    std::call_once(s.once, [&] {
        int major = 0, minor = 0;
        s.err = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (s.err == cudaSuccess) s.err = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        s.supported = (major == 10 && minor == 0);
        if (s.err == cudaSuccess) s.err = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (s.err == cudaSuccess && s.supported) s.err = cudaGetSymbolAddress(reinterpret_cast<void **>(&s.status), g_attn_status);
    });
    if (s.err != cudaSuccess) return ATTN_ERR_CUDA;
    if (!s.supported) return ATTN_ERR_UNSUPPORTED;
    *out = &s;
    return ATTN_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D map (col, row, slab) with a 128-byte swizzle; box = one 128-byte column group
// (64 bf16 or 32 fp32 elements) x box_rows rows x 1.  Strides are in elements.
// 3-D map (column, row, slab).  Loads use 64-column (128-byte) boxes with the
// 128-byte swizzle; the backward's output stores use 32 x 32 boxes with the 64-byte
// swizzle (box_cols = 32).
int make_map(CUtensorMap *m, const void *base, int d, long long rows, long long slabs, long long row_stride,
             long long slab_stride, int box_rows, bool fp32 = false, int box_cols = 0) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return ATTN_ERR_CUDA;
    const cuuint64_t esz = fp32 ? 4 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(slabs)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_stride) * esz, static_cast<cuuint64_t>(slab_stride) * esz};
    if (box_cols == 0) box_cols = fp32 ? 32 : 64;
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle swz = (box_cols * esz == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    CUresult r = enc(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D map over e4m3 bytes: `cols` bytes per row (contiguous), box {cols, box_rows, 1}
// with the 128-byte swizzle for 128-byte rows and the 64-byte swizzle for 64-byte rows.
int make_map_u8(CUtensorMap *m, const void *base, long long cols, long long rows, long long slabs,
                long long row_stride, long long slab_stride, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return ATTN_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(slabs)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_stride), static_cast<cuuint64_t>(slab_stride)};
    if (cols != 64 && cols != 128) return ATTN_ERR_UNSUPPORTED;
    cuuint32_t box[3] = {static_cast<cuuint32_t>(cols), static_cast<cuuint32_t>(box_rows), 1u};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

struct Shape {
    int B, H, N, d;
    long long total;  // packed token rows, or 0 for dense
    const int32_t *cu;
};

int map_for(CUtensorMap *m, const void *base, const Shape &s, int box_rows = 128, bool fp32 = false,
            int box_cols = 0) {
    if (s.cu)
        return make_map(m, base, s.d, s.total, s.H, static_cast<long long>(s.H) * s.d, s.d, box_rows, fp32, box_cols);
    return make_map(m, base, s.d, s.N, static_cast<long long>(s.B) * s.H, s.d, static_cast<long long>(s.N) * s.d,
                    box_rows, fp32, box_cols);
}

int check_common(const Shape &s, float scale) {
    if (s.B <= 0 || s.H <= 0 || s.N <= 0 || s.d <= 0) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (s.cu && s.total < 0) return ATTN_ERR_INVALID_ARG;
    if (s.d != 64 && s.d != 128) return ATTN_ERR_UNSUPPORTED;
    // grid limits: B <= 65535 (grid y), H <= 2^31-1, N/128 <= 65535 (grid z)
    if (s.B > 65535 || (s.N + 127) / 128 > 65535) return ATTN_ERR_UNSUPPORTED;
    // TMA extents are 32-bit
    if (s.cu ? s.total > 0x7fffffffLL : static_cast<long long>(s.B) * s.H > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

attn::Geom geom_of(const Shape &s, const uint8_t *key_keep, const uint8_t *block_mask = nullptr) {
    attn::Geom g{};
    g.block_mask = block_mask;
    g.nbt = (s.N + 127) / 128;
    g.B = s.B;
    g.H = s.H;
    g.N = s.N;
    g.d = s.d;
    g.varlen = s.cu != nullptr;
    g.cu_seqlens = s.cu;
    g.key_keep = key_keep;
    return g;
}

attn::SyncCtl ctl_of(DeviceState *ds) {
    attn::SyncCtl c{};
    c.status = ds->status;
    c.wait_limit_ns = static_cast<unsigned long long>(g_wait_limit_ms.load()) * 1000000ull;
    c.inject_skip_load = g_skip_load.load();
    c.inject_bad_tag = g_bad_tag.load();
    return c;
}

int fwd_impl(const void *q, const void *k, const void *v, void *o, float *lse, const Shape &s, float scale,
             int is_causal, const uint8_t *key_keep, void *stream, const uint8_t *block_mask = nullptr) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
    int rc = check_common(s, scale);
    if (rc) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_MISALIGNED;
    DeviceState *ds = nullptr;
    if ((rc = device_state(&ds))) return rc;
    if (s.cu && s.total == 0) return ATTN_OK;  // nothing to do
    attn::FwdLaunch a{};
    if ((rc = map_for(&a.tm_q, q, s)) || (rc = map_for(&a.tm_k, k, s)) || (rc = map_for(&a.tm_v, v, s)) ||
        (rc = map_for(&a.tm_o_st, o, s, 32, false, 32)))
        return rc;
    a.g = geom_of(s, key_keep, block_mask);
    a.ctl = ctl_of(ds);
    a.o = o;
    a.lse = lse;
    a.scale = scale;
    a.causal = is_causal ? 1 : 0;
    a.num_sms = ds->num_sms > 0 ? ds->num_sms : 1;
    return attn::launch_fwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int fwd_fp8_impl(const void *q, const void *k, const void *v, float q_scale, float k_scale, float v_scale, void *o,
                 float *lse, const Shape &s, float scale, int is_causal, const uint8_t *key_keep, void *stream,
                 const uint8_t *block_mask = nullptr) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
    int rc = check_common(s, scale);
    if (rc) return rc;
    for (float f : {q_scale, k_scale, v_scale})
        if (!(f > 0.f) || !std::isfinite(f)) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_MISALIGNED;
    DeviceState *ds = nullptr;
    if ((rc = device_state(&ds))) return rc;
    attn::FwdLaunch a{};
    if (s.cu && s.total == 0) return ATTN_OK;  // nothing to do
    // e4m3 maps with the bf16 maps' geometry (dense: slab b*H+h, row stride d; packed:
    // slab h, rows = tokens, row stride H*d), in bytes
    const long long rows = s.cu ? s.total : s.N, slabs = s.cu ? s.H : static_cast<long long>(s.B) * s.H;
    const long long rstride = s.cu ? static_cast<long long>(s.H) * s.d : s.d;
    const long long sstride = s.cu ? s.d : static_cast<long long>(s.N) * s.d;
    if ((rc = make_map_u8(&a.tm_q, q, s.d, rows, slabs, rstride, sstride, 128)) ||
        (rc = make_map_u8(&a.tm_k, k, s.d, rows, slabs, rstride, sstride, 128)) ||
        (rc = make_map_u8(&a.tm_v, v, s.d, rows, slabs, rstride, sstride, 128)) ||
        (rc = map_for(&a.tm_o_st, o, s, 32, false, 32)))
        return rc;
    a.g = geom_of(s, key_keep, block_mask);
    a.ctl = ctl_of(ds);
    a.o = o;
    a.lse = lse;
    a.scale = scale;
    a.causal = is_causal ? 1 : 0;
    a.num_sms = ds->num_sms > 0 ? ds->num_sms : 1;
    a.q_scale = q_scale;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    return attn::launch_fwd_fp8(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Deterministic backward: D and lse2 (fp32 each, one per query row and head), each
// region 256-byte aligned.
size_t bwd_ws_bytes(long long rows_x_heads, int /*d*/) { return 2 * up256(static_cast<size_t>(rows_x_heads) * 4); }

// Single-pass backward: the same two terms, then the fp32 dQ accumulator (d per row).
size_t fused_ws_bytes(long long rows_x_heads, int d) {
    return bwd_ws_bytes(rows_x_heads, d) + up256(static_cast<size_t>(rows_x_heads) * d * 4);
}

// phases: 7 = the deterministic backward's three kernels (bits 0-2), 56 = the
// single-pass backward's three kernels (bits 3-5); one bit = one kernel.
int bwd_impl(const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout,
             void *dq, void *dk, void *dv, const Shape &s, float scale, int is_causal, const uint8_t *key_keep,
             void *workspace, size_t workspace_bytes, void *stream, int phases,
             const uint8_t *block_mask = nullptr) {
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
    int rc = check_common(s, scale);
    if (rc) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return ATTN_ERR_MISALIGNED;
    const long long rows = s.cu ? s.total * s.H : static_cast<long long>(s.B) * s.H * s.N;
    const bool fused = (phases & 56) != 0;
    const size_t need = fused ? fused_ws_bytes(rows, s.d) : bwd_ws_bytes(rows, s.d);
    if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_MISALIGNED;
    DeviceState *ds = nullptr;
    if ((rc = device_state(&ds))) return rc;
    if (s.cu && s.total == 0) return ATTN_OK;
    attn::BwdLaunch a{};
    if ((rc = map_for(&a.tm_q, q, s)) || (rc = map_for(&a.tm_k, k, s)) || (rc = map_for(&a.tm_v, v, s)) ||
        (rc = map_for(&a.tm_do, dout, s)) || (rc = map_for(&a.tm_dk_st, dk, s, 32, false, 32)) ||
        (rc = map_for(&a.tm_dv_st, dv, s, 32, false, 32)))
        return rc;
    char *w = static_cast<char *>(workspace);
    if (fused) {
        a.dqacc = reinterpret_cast<float *>(w + bwd_ws_bytes(rows, s.d));
        if ((rc = map_for(&a.tm_dqacc, a.dqacc, s, 32, true, 32))) return rc;
    }
    a.g = geom_of(s, key_keep, block_mask);
    a.ctl = ctl_of(ds);
    a.o = o;
    a.dout = dout;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.dvec = reinterpret_cast<float *>(w);
    a.lse2 = reinterpret_cast<float *>(w + up256(static_cast<size_t>(rows) * 4));
    a.rows_total = rows;
    a.scale = scale;
    a.causal = is_causal ? 1 : 0;
    a.phases = phases;
    a.num_sms = ds->num_sms > 0 ? ds->num_sms : 1;
    const cudaError_t e = fused ? attn::launch_bwd_fused(a, static_cast<cudaStream_t>(stream))
                                : attn::launch_bwd(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

constexpr int kDeterministicPhases = 7;  // preprocess, dK/dV pass, dQ pass
constexpr int kFusedPhases = 56;         // preprocess + zeroing, single pass, dQ conversion

// Counter pairs of the dynamic unit deals, one per launch in flight: a launch takes the
// next pair round-robin and its last CTA returns the pair to zero.  A pair is reused
// only 1024 launches later; a device runs at most 128 kernels at once, and launches of
// one CUDA graph run in order, so two launches never hold the same pair together.
constexpr int kSchedSlots = 1024;
__device__ unsigned int g_sched_pool[kSchedSlots][2];

}  // namespace

int attn::forced_band() { return g_force_band.load(); }

unsigned int *attn::next_sched_slot() {
    static std::atomic<unsigned int> cursor{0};
    static std::atomic<unsigned int *> base[64];  // per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    unsigned int *b = base[dev].load();
    if (b == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_sched_pool) != cudaSuccess) return nullptr;
        b = static_cast<unsigned int *>(ptr);
        base[dev].store(b);
    }
    return b + 2 * (cursor.fetch_add(1u) % kSchedSlots);
}

extern "C" {

int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N, int d,
             float scale, int is_causal, const int32_t *cu_seqlens, void *stream) {
    Shape s{B, H, N, d, cu_seqlens ? static_cast<long long>(B) * N : 0, cu_seqlens};
    return fwd_impl(q, k, v, o, lse, s, scale, is_causal, nullptr, stream);
}

int attn_fwd_masked(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N, int d,
                    float scale, int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep, void *stream) {
    Shape s{B, H, N, d, cu_seqlens ? static_cast<long long>(B) * N : 0, cu_seqlens};
    return fwd_impl(q, k, v, o, lse, s, scale, is_causal, key_keep, stream);
}

int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse, int num_seqs, int total_tokens,
                    int max_seqlen, int H, int d, float scale, int is_causal, const int32_t *cu_seqlens,
                    const uint8_t *key_keep, void *stream) {
    if (!cu_seqlens) return ATTN_ERR_INVALID_ARG;
    Shape s{num_seqs, H, max_seqlen, d, total_tokens, cu_seqlens};
    return fwd_impl(q, k, v, o, lse, s, scale, is_causal, key_keep, stream);
}

int attn_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N,
                         int d, float scale, int is_causal, const uint8_t *block_mask, void *stream) {
    if (!block_mask) return ATTN_ERR_INVALID_ARG;
    if (N > 64 * 128) return ATTN_ERR_UNSUPPORTED;  // the kernels hold a row of the mask in 64 bits
    Shape s{B, H, N, d, 0, nullptr};
    return fwd_impl(q, k, v, o, lse, s, scale, is_causal, nullptr, stream, block_mask);
}

int attn_fwd_fp8(const void *q, const void *k, const void *v, float q_scale, float k_scale, float v_scale, void *o,
                 float *lse, int B, int H, int N, int d, float scale, int is_causal, void *stream) {
    Shape s{B, H, N, d, 0, nullptr};
    return fwd_fp8_impl(q, k, v, q_scale, k_scale, v_scale, o, lse, s, scale, is_causal, nullptr, stream);
}

int attn_fwd_fp8_masked(const void *q, const void *k, const void *v, float q_scale, float k_scale, float v_scale,
                        void *o, float *lse, int B, int H, int N, int d, float scale, int is_causal,
                        const uint8_t *key_keep, void *stream) {
    Shape s{B, H, N, d, 0, nullptr};
    return fwd_fp8_impl(q, k, v, q_scale, k_scale, v_scale, o, lse, s, scale, is_causal, key_keep, stream);
}

int attn_fwd_fp8_varlen(const void *q, const void *k, const void *v, float q_scale, float k_scale, float v_scale,
                        void *o, float *lse, int num_seqs, int total_tokens, int max_seqlen, int H, int d, float scale,
                        int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep, void *stream) {
    if (!cu_seqlens) return ATTN_ERR_INVALID_ARG;
    Shape s{num_seqs, H, max_seqlen, d, total_tokens, cu_seqlens};
    return fwd_fp8_impl(q, k, v, q_scale, k_scale, v_scale, o, lse, s, scale, is_causal, key_keep, stream);
}

int attn_fwd_fp8_blocksparse(const void *q, const void *k, const void *v, float q_scale, float k_scale,
                             float v_scale, void *o, float *lse, int B, int H, int N, int d, float scale,
                             int is_causal, const uint8_t *block_mask, void *stream) {
    if (!block_mask) return ATTN_ERR_INVALID_ARG;
    if (N > 64 * 128) return ATTN_ERR_UNSUPPORTED;  // the kernels hold a row of the mask in 64 bits
    Shape s{B, H, N, d, 0, nullptr};
    return fwd_fp8_impl(q, k, v, q_scale, k_scale, v_scale, o, lse, s, scale, is_causal, nullptr, stream, block_mask);
}

int attn_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o, const float *lse,
                         const void *dout, void *dq, void *dk, void *dv, int B, int H, int N, int d, float scale,
                         int is_causal, const uint8_t *block_mask, void *workspace, size_t workspace_bytes,
                         void *stream) {
    if (!block_mask) return ATTN_ERR_INVALID_ARG;
    if (N > 64 * 128) return ATTN_ERR_UNSUPPORTED;
    Shape s{B, H, N, d, 0, nullptr};
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, s, scale, is_causal, nullptr, workspace, workspace_bytes,
                    stream, kFusedPhases, block_mask);
}

size_t attn_bwd_workspace_bytes(int B, int H, int N, int d) {
    if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128)) return 0;
    return fused_ws_bytes(static_cast<long long>(B) * H * N, d);
}

size_t attn_bwd_deterministic_workspace_bytes(int B, int H, int N, int d) {
    if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128)) return 0;
    return bwd_ws_bytes(static_cast<long long>(B) * H * N, d);
}

int attn_bwd_deterministic(const void *q, const void *k, const void *v, const void *o, const float *lse,
                           const void *dout, void *dq, void *dk, void *dv, int B, int H, int N, int d, float scale,
                           int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep, void *workspace,
                           size_t workspace_bytes, void *stream) {
    Shape s{B, H, N, d, cu_seqlens ? static_cast<long long>(B) * N : 0, cu_seqlens};
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, s, scale, is_causal, key_keep, workspace, workspace_bytes,
                    stream, kDeterministicPhases);
}

size_t attn_bwd_varlen_workspace_bytes(int total_tokens, int H, int d) {
    if (total_tokens < 0 || H <= 0 || (d != 64 && d != 128)) return 0;
    return fused_ws_bytes(static_cast<long long>(total_tokens) * H, d);
}

int attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout, void *dq,
             void *dk, void *dv, int B, int H, int N, int d, float scale, int is_causal, const int32_t *cu_seqlens,
             const uint8_t *key_keep, void *workspace, size_t workspace_bytes, void *stream) {
    Shape s{B, H, N, d, cu_seqlens ? static_cast<long long>(B) * N : 0, cu_seqlens};
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, s, scale, is_causal, key_keep, workspace, workspace_bytes,
                    stream, kFusedPhases);
}

int attn_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout,
                    void *dq, void *dk, void *dv, int num_seqs, int total_tokens, int max_seqlen, int H, int d,
                    float scale, int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep, void *workspace,
                    size_t workspace_bytes, void *stream) {
    if (!cu_seqlens) return ATTN_ERR_INVALID_ARG;
    Shape s{num_seqs, H, max_seqlen, d, total_tokens, cu_seqlens};
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, s, scale, is_causal, key_keep, workspace, workspace_bytes,
                    stream, kFusedPhases);
}

int attn_bwd_phase(int phase, const void *q, const void *k, const void *v, const void *o, const float *lse,
                   const void *dout, void *dq, void *dk, void *dv, int num_seqs, int total_tokens, int max_seqlen,
                   int H, int d, float scale, int is_causal, const int32_t *cu_seqlens, const uint8_t *key_keep,
                   void *workspace, size_t workspace_bytes, void *stream) {
    if (phase < 0 || phase > 5) return ATTN_ERR_INVALID_ARG;
    Shape s{num_seqs, H, max_seqlen, d, cu_seqlens ? static_cast<long long>(total_tokens) : 0, cu_seqlens};
    return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, s, scale, is_causal, key_keep, workspace, workspace_bytes,
                    stream, 1 << phase);
}

int attn_status(void *stream) {
    DeviceState *ds = nullptr;
    int rc = device_state(&ds);
    if (rc) return rc;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, ds->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(ds->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return v;
}

const char *attn_strerror(int code) {
    switch (code) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument (null pointer, non-positive size or bad scale)";
        case ATTN_ERR_UNSUPPORTED: return "unsupported (head_dim must be 64 or 128; device must be sm_100)";
        case ATTN_ERR_MISALIGNED: return "a base pointer is not 16-byte aligned (workspace: 256-byte)";
        case ATTN_ERR_WORKSPACE: return "backward workspace missing or too small";
        case ATTN_ERR_CUDA: return "a CUDA call or kernel launch failed";
        case ATTN_ERR_TIMEOUT: return "a device-side pipeline wait exceeded its time limit";
        case ATTN_ERR_DEBUG_CHECK: return "a pipeline consistency check of the debug library failed";
        default: return "unknown status code";
    }
}

int attn_set_wait_limit_ms(int ms) {
    return g_wait_limit_ms.exchange(ms > 0 ? ms : 4000);
}

int attn_debug_ex2_poly(const float *x, float *y, long long n, void *stream) {
    if (!x || !y || n <= 0 || (n & 1)) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return ATTN_ERR_MISALIGNED;
    DeviceState *ds = nullptr;
    const int rc = device_state(&ds);
    if (rc) return rc;
    const long long pairs = n / 2;
    const unsigned blocks = static_cast<unsigned>(pairs / 256 + 1 < 4096 ? pairs / 256 + 1 : 4096);
    ex2_poly_probe_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float2 *>(x), reinterpret_cast<float2 *>(y), pairs);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_debug_skip_load(int load_index) {
    return g_skip_load.exchange(load_index < 0 ? -1 : load_index);
}

int attn_debug_force_band(int slices) { return g_force_band.exchange(slices > 0 ? slices : 0); }

int attn_debug_checks(void) { return attn::kDebugChecks ? 1 : 0; }

int attn_debug_corrupt_tag(int fill_index) { return g_bad_tag.exchange(fill_index < 0 ? -1 : fill_index); }

}  // extern "C"
