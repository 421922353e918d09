// attn_common.cuh -- parameter blocks and the bounded-wait / status machinery
// shared by the forward and backward kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

// LIBATTN_DEBUG=1 builds the debug library (libattn_debug.so): the same kernels with
// pipeline consistency checks that record ATTN_ERR_DEBUG_CHECK in the status word and
// stop the CTA the way an expired wait does (never a trap or an assert).
#ifndef LIBATTN_DEBUG
#define LIBATTN_DEBUG 0
#endif

namespace attn {

constexpr int kStatusOk = 0;
constexpr int kStatusUnsupported = 2;  // ATTN_ERR_UNSUPPORTED (a launch that cannot run as configured)
constexpr int kStatusTimeout = 6;      // ATTN_ERR_TIMEOUT
constexpr int kStatusDebugCheck = 7;   // ATTN_ERR_DEBUG_CHECK (debug library only)
constexpr bool kDebugChecks = LIBATTN_DEBUG != 0;

// Geometry of one (sequence, head) slice, common to dense and packed layouts.
// A tensor element (row r, column c) of slice (b, h) sits at
//   base + seq_off(b) + h * head_stride + r * row_stride + c
// Dense [B,H,N,d]:   seq_off = b*H*N*d, head_stride = N*d, row_stride = d.
// Packed [total,H,d]: seq_off = cu[b]*H*d, head_stride = d, row_stride = H*d.
// lse uses the same scheme with d = 1.
struct Geom {
    int B, H, N, d;
    int varlen;                 // 0 dense, 1 packed (cu_seqlens)
    const int32_t *cu_seqlens;  // device, B+1 entries (packed only)
    const uint8_t *key_keep;    // device, nullable
    const uint8_t *block_mask;  // device [H][nbt][nbt] tile mask (dense layout, nbt <= 64), nullable
    int nbt;                    // tiles per side of block_mask
    __device__ __forceinline__ void slice(int b, int &start, int &len) const {
        if (varlen) {
            start = cu_seqlens[b];
            len = cu_seqlens[b + 1] - start;
        } else {
            start = 0;
            len = N;
        }
    }
    // Element offset of (b, h, row 0, col 0) in a [.., d]-wide tensor.
    __device__ __forceinline__ long long base(int b, int h, int start, int width) const {
        if (varlen) return (static_cast<long long>(start) * H + h) * width;
        return (static_cast<long long>(b) * H + h) * static_cast<long long>(N) * width;
    }
    __device__ __forceinline__ long long row_stride(int width) const {
        return varlen ? static_cast<long long>(H) * width : width;
    }
    // Key-mask offset of key 0 of sequence b.
    __device__ __forceinline__ long long keep_base(int b, int start) const {
        return varlen ? start : static_cast<long long>(b) * N;
    }
    // TMA row coordinate of row 0 of (b, h): the maps are 3-D (col, row, slab).
    __device__ __forceinline__ int tma_row0(int start) const { return varlen ? start : 0; }
    __device__ __forceinline__ int tma_slab(int b, int h) const { return varlen ? h : b * H + h; }
};

// A set of 128-row tiles [lo, hi) of one unit's sweep, all of them or (with a tile
// mask) those whose bit is set.  next(x) is the first member >= x, or hi.
struct TileSet {
    uint64_t bits;  // members (only with a tile mask; then hi <= 64)
    int lo, hi;
    bool sparse;
    __device__ __forceinline__ int next(int x) const {
        if (!sparse) return x < hi ? max(x, lo) : hi;
        if (x >= hi) return hi;
        const uint64_t m = bits & (~0ull << x);
        return m ? min(__ffsll(static_cast<long long>(m)) - 1, hi) : hi;
    }
    __device__ __forceinline__ bool has(int x) const {
        return x >= lo && x < hi && (!sparse || ((bits >> x) & 1ull));
    }
    __device__ __forceinline__ int count() const { return sparse ? __popcll(bits) : max(0, hi - lo); }
    __device__ __forceinline__ int last() const {  // largest member, or lo - 1 if none
        if (!sparse) return hi - 1;
        return bits ? 63 - __clzll(static_cast<long long>(bits)) : lo - 1;
    }
};

// Key tiles [0, n) of query tile qt that head h attends (SP: a tile mask is given;
// a compile-time flag, so that kernels without one carry none of this).
template <bool SP>
__device__ __forceinline__ TileSet row_tiles(const Geom &g, int h, int qt, int n) {
    TileSet t{0ull, 0, n, SP};
    if (SP) {
        const uint8_t *r = g.block_mask + (static_cast<long long>(h) * g.nbt + qt) * g.nbt;
        for (int j = 0; j < n; ++j) t.bits |= static_cast<uint64_t>(r[j] != 0) << j;
    }
    return t;
}

// Query tiles [lo, n) that attend key tile kt of head h.
template <bool SP>
__device__ __forceinline__ TileSet col_tiles(const Geom &g, int h, int kt, int lo, int n) {
    TileSet t{0ull, lo, n, SP};
    if (SP) {
        const uint8_t *c = g.block_mask + static_cast<long long>(h) * g.nbt * g.nbt + kt;
        for (int i = lo; i < n; ++i) t.bits |= static_cast<uint64_t>(c[static_cast<long long>(i) * g.nbt] != 0) << i;
    }
    return t;
}

// Rank r of a persistent schedule over `units` work units per (sequence, head) slice
// and BH slices, as (unit index k, slice bh).  The slices are taken in bands of
// `band` (the last band may be smaller) and, inside a band, unit index first: ranks
// 0, 1, ... are the first units of every slice of band 0, then their second units,
// and so on.  With unit index 0 the heaviest, this is heaviest first within a band,
// while the CTAs running at any one time share the data of one or two bands (their
// K/V, or Q/dO/dQ), which the host sizes to fit the L2 cache.  band = BH: unit index
// first over all slices.
__device__ __forceinline__ void rank_to_unit(int r, int units, int BH, int band, int &k, int &bh) {
    const int per_band = band * units;
    const int bnd = r / per_band;
    const int rr = r - bnd * per_band;
    const int nb = min(band, BH - bnd * band);
    k = rr / nb;
    bh = bnd * band + (rr - k * nb);
}

// Slices per band for rank_to_unit: all of them unless their data exceeds four times
// the L2 cache, then as many as fill about half of it (at least one).  Measured: with
// the backward's Q/dO/dQ at 830 MB (8 packed sequences of up to 3,141 tokens, 32
// heads) bands of 19 slices cut the time by 19 %; at 68-135 MB (B4 H16 N2048 d64,
// B2 H16 N4096 d128) banding only unbalanced the last band (+15 %), and the forward,
// whose two query tiles share each K/V load, lost 22 % at 410 MB.
__host__ __forceinline__ int l2_band(int BH, double bytes_per_slice, double band_above = 512.0 * 1024 * 1024) {
    constexpr double kBudget = 64.0 * 1024 * 1024;  // about half of the 126 MB L2
    if (BH * bytes_per_slice <= band_above) return BH;
    const int b = static_cast<int>(kBudget / bytes_per_slice);
    return b < 1 ? 1 : (b > BH ? BH : b);
}

struct SyncCtl {
    int *status;             // device status word (first error wins)
    unsigned long long wait_limit_ns;
    int inject_skip_load;    // test hook: index of a pipeline load to skip, or -1
    int inject_bad_tag;      // test hook (debug library): ring fill whose check tag is written wrong, or -1
};

// Record an error once and raise the CTA-wide abort flag.
__device__ __forceinline__ void raise_abort(const SyncCtl &ctl, volatile int *abort_flag, int code) {
    atomicCAS(ctl.status, 0, code);
    *abort_flag = 1;
    __threadfence_block();
}

// Debug library: a waiter that has just seen phase k of `bar` complete must find phase
// k+1 still open.  Every barrier here is built so that its next phase needs an action
// that follows this wait (the waiter's own arrive, or a release it gates), so a
// completed k+1 means a producer ran two phases ahead of a consumer: the parity
// protocol can no longer tell the phases apart.  Release library: always true.
__device__ __forceinline__ bool phase_consistent(uint32_t bar, uint32_t parity, const SyncCtl &ctl,
                                                 volatile int *abort_flag) {
    if constexpr (kDebugChecks) {
        if (mbar_test_wait(bar, parity ^ 1u)) {
            raise_abort(ctl, abort_flag, kStatusDebugCheck);
            return false;
        }
    }
    return true;
}

// Bounded wait on an mbarrier phase.  Returns false (and raises the abort flag on
// expiry) if the wait gave up, either because the limit passed or because another
// role of the CTA already aborted.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, const SyncCtl &ctl,
                                           volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return phase_consistent(bar, parity, ctl, abort_flag);
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return phase_consistent(bar, parity, ctl, abort_flag);
        if ((it & 15u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > ctl.wait_limit_ns) {
                raise_abort(ctl, abort_flag, kStatusTimeout);
                return false;
            }
        }
    }
}

// Bounded wait used during teardown: ignores the abort flag (the hardware must be
// drained before shared memory / tensor memory are released), still time-limited.
__device__ __forceinline__ bool drain_phase(uint32_t bar, uint32_t parity, const SyncCtl &ctl,
                                            volatile int *abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0 && globaltimer_ns() - t0 > ctl.wait_limit_ns) {
            raise_abort(ctl, abort_flag, kStatusTimeout);
            return false;
        }
    }
}

// One warp writes a 32-row x 32-column bf16 block to global memory.  On entry lane
// r holds row r as 16 packed words (the tensor-memory layout: one row per lane).
// Stored directly, every warp store would touch 32 rows, 16 bytes each; instead
// the block passes through a 2 KB shared-memory staging area so that each store
// instruction writes 8 rows x 64 contiguous bytes.  Chunk c (16 bytes) of row r
// sits at r*64 + ((c ^ (r >> 1)) & 3)*16, which keeps both the row-per-lane writes
// and the 4-lanes-per-row reads free of bank conflicts.  Rows r >= nvalid are not
// written.  dst0 points at column 0 of row 0; ld is the row stride in elements.
__device__ __forceinline__ void warp_store_rows32(uint32_t stage, const uint32_t (&pk)[16], __nv_bfloat16 *dst0,
                                                  long long ld, int nvalid, int lane) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
        st_shared_v4(stage + lane * 64 + (((c ^ (lane >> 1)) & 3) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                     pk[4 * c + 3]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = i * 8 + (lane >> 2), c = lane & 3;
        const uint4 v = ld_shared_v4(stage + r * 64 + (((c ^ (r >> 1)) & 3) << 4));
        if (r < nvalid) *reinterpret_cast<uint4 *>(dst0 + r * ld + c * 8) = v;
    }
    __syncwarp();  // the staging area is free again
}

}  // namespace attn
