// attn_bwd_sm100.cu -- exact-attention backward for B200 (sm_100a).
//
// The backward recomputes the probabilities from Q, K and the forward's
// logsumexp instead of storing them ("4.5 注意力优化实战：从PyTorch到CUDA的完整流程",
// 第四步 §2: dQ sweeps the key/value blocks, dK and dV sweep the query blocks, and
// the softmax normaliser saved by the forward is reused).  With P the softmax
// probabilities and dO the upstream gradient:
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - D),  D_i = sum_c dO_ic O_ic,
//   dQ = scale dS K,   dK = scale dS^T Q.
// (D_i equals sum_k P_ik dP_ik because O_i = sum_k P_ik V_k.)
//
// Three launches on one stream, with no atomics (the result is deterministic):
//   1. attn_bwd_pre_kernel   D_i and lse2_i = lse_i log2(e) (+inf for rows that saw
//                            no key, so their recomputed P is exactly 0).
//   2. attn_bwd_dkdv_sm100_kernel: work unit = one 128-key tile of one (b, h), which
//      sweeps the 128-row query tiles (from the diagonal when causal):
//        S^T  = K_j Q_i^T   (SS, M=128 keys, N=128 queries)   -> TMEM
//        dP^T = V_j dO_i^T  (SS)                              -> TMEM
//        P^T  = 2^(S^T scale log2e - lse2)  written back over S^T as bf16,
//        dS^T = P^T o (dP^T - D)            written back over dP^T as bf16
//               (8 warps; each keeps its P in fp32 registers for dS)
//        dV  += P^T dO_i    (TS: A = P^T from TMEM, M=128, N=d, K=128)
//        dK  += dS^T Q_i    (TS: A = dS^T from TMEM)
//      then writes dV and scale*dK.
//   3. attn_bwd_dq_sm100_kernel: work unit = one 128-row query tile of one (b, h),
//      which sweeps the key tiles:
//        S  = Q_i K_j^T, dP = dO_i V_j^T (SS, M=128 queries, N=128 keys) -> TMEM,
//        S double-buffered so the next tile's product overlaps this tile's math;
//        dS = P o (dP - D) written back over S as bf16 (8 warps);
//        dQ += dS K_j      (TS: A = dS from TMEM, M=128, N=d, K=128)
//      then writes scale*dQ.
// Both main kernels are persistent (one CTA per SM, units dealt heaviest first in a
// snake order).  Every barrier keeps counting phases across units, so a CTA loads
// the next unit's tiles and issues its first products while the math warps are
// still writing the previous unit's result.
// Every product is a full 128 x 128 (x d) tensor-core tile; the extra S and dP
// products of the dQ pass cost less than the reductions they replace.
// With a tile mask (block-sparse attention, the SP instantiations) a unit sweeps only
// the partner tiles the mask keeps; a unit left with none writes zeros and computes
// nothing.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "attn_common.cuh"
#include "attn_launch.h"

namespace attn {

constexpr float kLog2e = 1.4426950408889634f;

// ============================================================================ preprocess
// One row of d elements per (d/8) threads (16 bytes of O and of dO each); a CTA
// covers kPrePasses passes of 256 / (d/8) consecutive rows, whose loads are all
// issued before any is used, so that each thread keeps several loads in flight (the
// kernel is HBM-bound).  Rows are in the lse layout order, which is
// also the row order of the flat [rows, d] view of O and dO.
constexpr int kPrePasses = 4;
// With a non-null dqacc (the single-pass backward) the kernel also zeroes the fp32 dQ
// accumulator's rows (same flat [rows, d] order), which the fused kernel then adds into.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(const __nv_bfloat16 *__restrict__ o,
                                                          const __nv_bfloat16 *__restrict__ dout,
                                                          const float *__restrict__ lse, float *__restrict__ dvec,
                                                          float *__restrict__ lse2, float *__restrict__ dqacc,
                                                          long long rows, const int32_t *cu_seqlens, int nseq, int H) {
    constexpr int TPR = D / 8;          // threads per row
    constexpr int RPP = 256 / TPR;      // rows per pass
    long long limit = rows;
    if (cu_seqlens) limit = min(rows, static_cast<long long>(cu_seqlens[nseq]) * H);
    const int part = threadIdx.x % TPR;
    const long long row0 = static_cast<long long>(blockIdx.x) * (RPP * kPrePasses) + threadIdx.x / TPR;
    uint4 a[kPrePasses], g[kPrePasses];
#pragma unroll
    for (int u = 0; u < kPrePasses; ++u) {
        const long long row = row0 + u * RPP;
        if (row < limit) {
            a[u] = *reinterpret_cast<const uint4 *>(o + row * D + part * 8);
            g[u] = *reinterpret_cast<const uint4 *>(dout + row * D + part * 8);
        } else {
            a[u] = make_uint4(0u, 0u, 0u, 0u);
            g[u] = a[u];
        }
    }
#pragma unroll
    for (int u = 0; u < kPrePasses; ++u) {
        const long long row = row0 + u * RPP;
        const uint32_t aw[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, gw[4] = {g[u].x, g[u].y, g[u].z, g[u].w};
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = unpack_bf16x2(aw[e]);
            const float2 y = unpack_bf16x2(gw[e]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
#pragma unroll
        for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (row < limit && part == 0) {
            dvec[row] = acc;
            const float L = lse[row];
            lse2[row] = (L == -INFINITY) ? INFINITY : L * kLog2e;
        }
        if (dqacc != nullptr && row < limit) {
            float4 *z = reinterpret_cast<float4 *>(dqacc + row * D + part * 8);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = z[0];
        }
    }
}

struct BwdParams {
    Geom g;
    SyncCtl ctl;
    __nv_bfloat16 *dq, *dk, *dv;
    const float *dvec, *lse2;
    float scale;
    float scale_log2;
    int causal;
    int n_tiles;  // 128-row tiles per slice
};

// Offset of K-step kk (16 columns) inside a 128-row, 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t kstep_off(int kk) { return (kk >> 2) * 16384 + (kk & 3) * 32; }

// ============================================================================ persistent schedule
// Both backward passes run one persistent CTA per SM.  Work units are ranked
// heaviest first (for causal masking: key tile 0 / the last query tile have the
// most partner tiles); CTA c of G takes ranks c, 2G-1-c, 2G+c, 4G-1-c, ... (a
// snake order, which balances the per-CTA totals of a decreasing sequence).  Every
// role of a CTA walks the same list, so they agree on the tiles without talking.
__device__ __forceinline__ int snake_rank(int k, int c, int G) { return k * G + ((k & 1) ? (G - 1 - c) : c); }

// ============================================================================ dK / dV
template <int D>
struct DkdvCfg {
    static constexpr int kTile = 128 * D * 2;  // any 128-row bf16 tile (K, V, Q, dO)
    static constexpr int kBoxes = D / 64;
    static constexpr int kStages = 2;
    static constexpr int kThreads = 320;
    static constexpr int kTmemCols = 512;
    static constexpr int kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static constexpr int kOffK = 0, kOffV = kTile;
    static constexpr int kOffQ = 2 * kTile;                  // + st * kTile
    static constexpr int kOffDO = kOffQ + kStages * kTile;   // + st * kTile
    static constexpr int kOffVec = kOffDO + kStages * kTile; // + st * 1024: lse2[128], D[128]
    static constexpr int kOffStage = kOffVec + kStages * 1024;  // 8 math warps x 2 KB output staging
    static constexpr int kOffBar = kOffStage + 8 * 2048;
    static constexpr int kBarKVFull = 0;
    static constexpr int kBarKVEmpty = 1;                // K_j, V_j free: the tile's last S^T/dP^T are done
    static constexpr int kBarQFull = 2;                  // + st
    static constexpr int kBarQEmpty = 2 + kStages;       // + st
    static constexpr int kBarSFull = 2 + 2 * kStages;
    static constexpr int kBarDPFull = 3 + 2 * kStages;
    static constexpr int kBarPFull = 4 + 2 * kStages;    // P^T written (256 threads)
    static constexpr int kBarDSFull = 5 + 2 * kStages;   // dS^T written (256 threads)
    static constexpr int kBarKdv = 6 + 2 * kStages;      // dV, dK accumulators complete
    static constexpr int kBarAccFree = 7 + 2 * kStages;  // dV, dK copied out of TMEM (256 threads)
    static constexpr int kBarDone = 8 + 2 * kStages;
    static constexpr int kNumBars = 9 + 2 * kStages;
    static constexpr int kSmemBytes = 1024 + kOffBar + kNumBars * 8 + 16;
    static_assert(kTile % 1024 == 0, "swizzled tiles must be 1024-byte aligned");
    static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-CTA shared-memory limit");
};

template <int D, bool SP>
__device__ __forceinline__ void dkdv_persistent(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                                const CUtensorMap &tm_v, const CUtensorMap &tm_do,
                                                const CUtensorMap &tm_dk_st, const CUtensorMap &tm_dv_st,
                                                const BwdParams &p, uint8_t *smem_raw) {
    using C = DkdvCfg<D>;
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    uint8_t *sptr = smem_raw + (sbase - raw_u32);
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sptr + C::kOffBar + C::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
    const int BH = p.g.B * p.g.H;
    const int T = BH * p.n_tiles;
    // work unit of rank r: key tile j (heaviest = 0), slice (b, h); false if empty.
    // qs: the query tiles that attend key tile j (all from i0 on without a tile
    // mask); nq of them, walked in increasing order.
    struct Tile {
        int b, h, j, start, len, kv0, i0, nq;
        TileSet qs;
    };
    auto tile_at = [&](int r, Tile &t) -> bool {
        t.j = r / BH;
        const int bh = r - t.j * BH;
        t.b = bh / p.g.H;
        t.h = bh - t.b * p.g.H;
        p.g.slice(t.b, t.start, t.len);
        t.kv0 = t.j * 128;
        if (t.kv0 >= t.len) return false;
        t.i0 = p.causal ? t.j : 0;
        t.qs = col_tiles<SP>(p.g, t.h, t.j, t.i0, (t.len + 127) / 128);
        t.nq = t.qs.count();
        return true;
    };

    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i)
            mbar_init(bar(i), (i == C::kBarPFull || i == C::kBarDSFull || i == C::kBarAccFree) ? 256u : 1u);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    int n_q = 0, n_kv = 0;  // loader: query-tile and K/V loads started (for the abort drain)

    if (warp == 8) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
        }
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int r = snake_rank(k, cta, G);
            if (r >= T) break;
            Tile t;
            if (!tile_at(r, t) || t.nq == 0) continue;  // (nq == 0: the math warps write zeros)
            const int row0 = p.g.tma_row0(t.start), slab = p.g.tma_slab(t.b, t.h);
            const long long lrow0 = p.g.base(t.b, t.h, t.start, 1), lrs = p.g.row_stride(1);
            // K_j, V_j once the previous tile's last S^T / dP^T have read theirs
            ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarKVEmpty), (n_kv & 1) ^ 1, p.ctl, abort_flag));
            if (!ok) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(C::kBarKVFull), 2 * C::kTile);
#pragma unroll
                for (int x = 0; x < C::kBoxes; ++x) {
                    tma_load_3d(sbase + C::kOffK + x * 16384, &tm_k, bar(C::kBarKVFull), x * 64, row0 + t.kv0, slab);
                    tma_load_3d(sbase + C::kOffV + x * 16384, &tm_v, bar(C::kBarKVFull), x * 64, row0 + t.kv0, slab);
                }
            }
            ++n_kv;
            for (int it = 0, i = t.qs.next(t.i0); it < t.nq; ++it, i = t.qs.next(i + 1)) {
                const int gi = n_q, st = gi % C::kStages;
                ok = __all_sync(0xffffffffu,
                                wait_phase(bar(C::kBarQEmpty + st), ((gi / C::kStages) & 1) ^ 1, p.ctl, abort_flag));
                if (!ok) break;
                const int q0 = i * 128;
                float *vec = reinterpret_cast<float *>(sptr + C::kOffVec + st * 1024);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int q = q0 + u * 32 + lane;
                    float l2 = INFINITY, dd = 0.f;  // rows past the sequence: P = 0
                    if (q < t.len) {
                        l2 = p.lse2[lrow0 + q * lrs];
                        dd = p.dvec[lrow0 + q * lrs];
                    }
                    vec[u * 32 + lane] = l2;
                    vec[128 + u * 32 + lane] = dd;
                }
                __syncwarp();
                if (lane == 0 && gi != p.ctl.inject_skip_load) {  // (test hook: this stage never fills)
                    mbar_arrive_expect_tx(bar(C::kBarQFull + st), 2 * C::kTile);
#pragma unroll
                    for (int x = 0; x < C::kBoxes; ++x) {
                        tma_load_3d(sbase + C::kOffQ + st * C::kTile + x * 16384, &tm_q, bar(C::kBarQFull + st),
                                    x * 64, row0 + q0, slab);
                        tma_load_3d(sbase + C::kOffDO + st * C::kTile + x * 16384, &tm_do, bar(C::kBarQFull + st),
                                    x * 64, row0 + q0, slab);
                    }
                }
                ++n_q;
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
            constexpr uint32_t idKV = idesc_bf16_f32(128, D, 0, 1);   // dV, dK
            // P^T / dS^T sit in TMEM with queries 0-63 at columns 0-31 and queries
            // 64-127 at columns 64-95 of the S^T / dP^T regions (each math warp writes
            // only inside the columns it read).
            auto acol = [](int kk) -> uint32_t { return kk < 4 ? kk * 8 : 64 + (kk - 4) * 8; };
            auto issue_s = [&](int gi) {
                const uint32_t qs = sbase + C::kOffQ + (gi % C::kStages) * C::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::kColS, sw128_desc(sbase + C::kOffK + kstep_off(kk), 16, 1024),
                           sw128_desc(qs + kstep_off(kk), 16, 1024), idS, kk > 0);
                tc_commit(bar(C::kBarSFull));
            };
            auto issue_dp = [&](int gi) {
                const uint32_t ds = sbase + C::kOffDO + (gi % C::kStages) * C::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::kColDP, sw128_desc(sbase + C::kOffV + kstep_off(kk), 16, 1024),
                           sw128_desc(ds + kstep_off(kk), 16, 1024), idS, kk > 0);
                tc_commit(bar(C::kBarDPFull));
            };
            auto wait_q = [&](int gi) {
                return wait_phase(bar(C::kBarQFull + gi % C::kStages), (gi / C::kStages) & 1, p.ctl, abort_flag);
            };
            bool ok = true;
            int gbase = 0, n_t = 0;
            for (int k = 0; ok; ++k) {
                const int r = snake_rank(k, cta, G);
                if (r >= T) break;
                Tile t;
                if (!tile_at(r, t) || t.nq == 0) continue;
                ok = wait_phase(bar(C::kBarKVFull), n_t & 1, p.ctl, abort_flag);
                if (ok) ok = wait_q(gbase);
                if (!ok) break;
                tc_fence_after();
                // S^T / dP^T regions are free: the previous tile's last dV / dK, which
                // read P^T / dS^T from them, were issued earlier (in-order completion)
                // and its math warps had finished reading before those were issued.
                issue_s(gbase);
                issue_dp(gbase);
                if (t.nq == 1) tc_commit(bar(C::kBarKVEmpty));
                for (int it = 0; ok && it < t.nq; ++it) {
                    const int gi = gbase + it, st = gi % C::kStages;
                    const uint32_t qs = sbase + C::kOffQ + st * C::kTile;
                    const uint32_t dos = sbase + C::kOffDO + st * C::kTile;
                    const bool more = it + 1 < t.nq;
                    // dV += P^T dO_i   (K = 128 queries: 8 steps)
                    ok = wait_phase(bar(C::kBarPFull), gi & 1, p.ctl, abort_flag);
                    if (ok && it == 0 && n_t > 0)  // the previous tile's dV / dK have been copied out
                        ok = wait_phase(bar(C::kBarAccFree), (n_t - 1) & 1, p.ctl, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + C::kColDV, tmem + C::kColS + acol(kk), sw128_desc(dos + kk * 2048, 16384, 1024),
                               idKV, (it > 0 || kk > 0) ? 1u : 0u);
                    // S^T_{i+1} may overwrite P^T_i now: the math warps keep P in registers
                    // and dV_i, issued first, completes first.
                    if (more) {
                        ok = wait_q(gi + 1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(gi + 1);
                    }
                    // dK += dS^T Q_i
                    ok = wait_phase(bar(C::kBarDSFull), gi & 1, p.ctl, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + C::kColDK, tmem + C::kColDP + acol(kk), sw128_desc(qs + kk * 2048, 16384, 1024),
                               idKV, (it > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar(C::kBarQEmpty + st));
                    if (more) {
                        issue_dp(gi + 1);
                        if (it + 2 == t.nq) tc_commit(bar(C::kBarKVEmpty));  // last S^T / dP^T of the tile
                    }
                }
                if (!ok) break;
                tc_commit(bar(C::kBarKdv));
                gbase += t.nq;
                ++n_t;
            }
            tc_commit(bar(C::kBarDone));
            drain_phase(bar(C::kBarDone), 0, p.ctl, abort_flag);
        }
    } else {
        // ------------------------------------------------------------ P^T and dS^T (warps 0-7)
        // warp w: key rows 32*(w%4).., query columns 64*(w/4) .. +63 of each query tile.
        const int q4 = warp & 3, hf = warp >> 2;
        const int kr = q4 * 32 + lane;  // key row within the tile
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::kColS + hf * 64;
        const uint32_t tDP = tmem + lane_off + C::kColDP + hf * 64;
        const float c2 = p.scale_log2;
        bool ok = true;
        int gbase = 0, n_t = 0;
        for (int k = 0; ok; ++k) {
            const int r = snake_rank(k, cta, G);
            if (r >= T) break;
            Tile t;
            if (!tile_at(r, t)) continue;
            const int key = t.kv0 + kr;
            if (t.nq == 0) {
                // The tile mask leaves key tile j no query tile: dV = dK = 0 for its keys
                // (warps 0-3 write dV, 4-7 dK), and nothing was computed.
                if (key < t.len) {
                    uint4 *dst = reinterpret_cast<uint4 *>((hf == 0 ? p.dv : p.dk) + p.g.base(t.b, t.h, t.start, D) +
                                                           static_cast<long long>(key) * p.g.row_stride(D));
#pragma unroll 1
                    for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                }
                continue;
            }
            bool kvalid = key < t.len;
            if (kvalid && p.g.key_keep) kvalid = p.g.key_keep[p.g.keep_base(t.b, t.start) + key] != 0;
            for (int it = 0, i = t.qs.next(t.i0); it < t.nq; ++it, i = t.qs.next(i + 1)) {
                const int gi = gbase + it, st = gi % C::kStages;
                ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarSFull), gi & 1, p.ctl, abort_flag));
                if (ok)
                    ok = __all_sync(0xffffffffu,
                                    wait_phase(bar(C::kBarQFull + st), (gi / C::kStages) & 1, p.ctl, abort_flag));
                if (!ok) break;
                tc_fence_after();
                const float4 *vec = reinterpret_cast<const float4 *>(sptr + C::kOffVec + st * 1024) + hf * 16;
                uint32_t sr[2][32];
                tmem_ld32(tS, sr[0]);
                tmem_ld32(tS + 32, sr[1]);
                tmem_wait_ld();
                // P^T = 2^(S^T c - lse2), 0 where the query precedes the key (causal),
                // for keys outside the sequence or padded, and for rows past the end.
                const int qb = i * 128 + hf * 64;  // first query column of this warp
                int lim = p.causal ? key - qb : 0;            // columns c < lim are masked
                if (!kvalid) lim = 64;
                float pf[64];
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 l2 = vec[c4];
                    const float l2v[4] = {l2.x, l2.y, l2.z, l2.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = c4 * 4 + e;
                        pf[c] = ex2_approx(fmaf(__uint_as_float(sr[c >> 5][c & 31]), c2, -l2v[e]));
                    }
                }
                if (lim > 0) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c < lim) pf[c] = 0.f;
                }
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pf[x * 32 + 2 * c], pf[x * 32 + 2 * c + 1]);
                    tmem_st16(tS + x * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(C::kBarPFull));
                // dS^T = P^T o (dP^T - D), P taken from registers (fp32)
                ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarDPFull), gi & 1, p.ctl, abort_flag));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    uint32_t dr[32];
                    tmem_ld32(tDP + x * 32, dr);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 dd = vec[32 + x * 8 + c4];
                        const int c = x * 32 + c4 * 4;
                        pk[2 * c4] = pack_bf16x2(pf[c] * (__uint_as_float(dr[c4 * 4]) - dd.x),
                                                 pf[c + 1] * (__uint_as_float(dr[c4 * 4 + 1]) - dd.y));
                        pk[2 * c4 + 1] = pack_bf16x2(pf[c + 2] * (__uint_as_float(dr[c4 * 4 + 2]) - dd.z),
                                                     pf[c + 3] * (__uint_as_float(dr[c4 * 4 + 3]) - dd.w));
                    }
                    tmem_st16(tDP + x * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(C::kBarDSFull));
            }
            if (!ok) break;
            // ---- epilogue: warps 0-3 write dV, warps 4-7 write scale * dK; TMEM is
            // released (acc free) as soon as the values are in registers
            ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarKdv), n_t & 1, p.ctl, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const bool is_dv = hf == 0;
            const int key_w0 = t.kv0 + q4 * 32;  // this warp's first key row
            __nv_bfloat16 *out0 = (is_dv ? p.dv : p.dk) + p.g.base(t.b, t.h, t.start, D) +
                                  static_cast<long long>(key_w0) * p.g.row_stride(D);
            const float mul = is_dv ? 1.f : p.scale;
            const uint32_t col = is_dv ? C::kColDV : C::kColDK;
            const uint32_t stage = sbase + C::kOffStage + warp * 2048;
            // A full 32-row block goes out by TMA store from the stage (its layout is
            // the 64-byte swizzle of a 32 x 32 box), so the warp does not wait for the
            // global writes; a block reaching past the sequence's end (which a packed
            // layout could not clip) is written row by row.
            const bool by_tma = t.len - key_w0 >= 32;
            const CUtensorMap *tm_out = is_dv ? &tm_dv_st : &tm_dk_st;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t rr[32];
                tmem_ld32(tmem + lane_off + col + c0, rr);
                tmem_wait_ld();
                if (c0 + 32 == D) {
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarAccFree));
                }
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    pk[c] = pack_bf16x2(__uint_as_float(rr[2 * c]) * mul, __uint_as_float(rr[2 * c + 1]) * mul);
                if (by_tma) {
                    if (lane == 0) bulk_wait_read0();  // the previous store has read the stage
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        st_shared_v4(stage + lane * 64 + (((c ^ (lane >> 1)) & 3) << 4), pk[4 * c], pk[4 * c + 1],
                                     pk[4 * c + 2], pk[4 * c + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(tm_out, stage, c0, p.g.tma_row0(t.start) + key_w0, p.g.tma_slab(t.b, t.h));
                        bulk_commit();
                    }
                } else {
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
                    warp_store_rows32(stage, pk, out0 + c0, p.g.row_stride(D), t.len - key_w0, lane);
                }
            }
            gbase += t.nq;
            ++n_t;
        }
        if (lane == 0) bulk_wait0();  // this warp's output stores are complete
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 8 && lane == 0 && *abort_flag) {
        // After an abort, every copy the loader started must land before the CTA exits.
        if (n_kv > 0) drain_phase(bar(C::kBarKVFull), (n_kv - 1) & 1, p.ctl, abort_flag);
        for (int gi = max(0, n_q - C::kStages); gi < n_q; ++gi)
            if (gi != p.ctl.inject_skip_load)
                drain_phase(bar(C::kBarQFull + gi % C::kStages), (gi / C::kStages) & 1, p.ctl, abort_flag);
    }
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ============================================================================ dQ
template <int D>
struct DqCfg {
    static constexpr int kTile = 128 * D * 2;
    static constexpr int kBoxes = D / 64;
    // K_j is read by S_j and by dQ_j (the last product of step j), V_j only by dP_j,
    // so K gets the deeper ring: the next tiles' loads are in flight a full step ahead.
    static constexpr int kKStages = (D == 128) ? 3 : 6;
    static constexpr int kVStages = (D == 128) ? 2 : 4;
    static constexpr int kThreads = 320;
    static constexpr int kTmemCols = 512;
    static constexpr int kColS0 = 0, kColS1 = 128, kColDP = 256, kColDQ = 384;
    static constexpr int kOffQ = 0, kOffDO = kTile;
    static constexpr int kOffK = 2 * kTile;                     // + s * kTile
    static constexpr int kOffV = kOffK + kKStages * kTile;      // + s * kTile
    static constexpr int kOffBar = kOffV + kVStages * kTile;
    static constexpr int kBarQFull = 0;                          // Q_i, dO_i of the tile loaded
    static constexpr int kBarQEmpty = 1;                         // the tile's last S / dP are done
    static constexpr int kBarKFull = 2;                          // + slot
    static constexpr int kBarKEmpty = kBarKFull + kKStages;      // + slot
    static constexpr int kBarVFull = kBarKEmpty + kKStages;      // + slot
    static constexpr int kBarVEmpty = kBarVFull + kVStages;      // + slot
    static constexpr int kBarSFull = kBarVEmpty + kVStages;      // + buffer
    static constexpr int kBarDPFull = kBarSFull + 2;
    static constexpr int kBarDPFree = kBarDPFull + 1;            // 256 threads copied dP out
    // 256 threads wrote dS, + buffer: per buffer, so that the math warps (which may
    // finish step j+1 before the issuer looks at step j) never run two phases ahead
    static constexpr int kBarDSFull = kBarDPFree + 1;
    static constexpr int kBarDq = kBarDSFull + 2;                // dQ accumulator complete
    static constexpr int kBarAccFree = kBarDq + 1;               // dQ copied out of TMEM (256 threads)
    static constexpr int kBarDone = kBarAccFree + 1;
    static constexpr int kNumBars = kBarDone + 1;
    static constexpr int kSmemBytes = 1024 + kOffBar + kNumBars * 8 + 16;
    static_assert(kTile % 1024 == 0, "swizzled tiles must be 1024-byte aligned");
    static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-CTA shared-memory limit");
    static_assert(kColDQ + D <= kTmemCols, "tensor memory budget");
};

template <int D, bool SP>
__device__ __forceinline__ void dq_persistent(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                              const CUtensorMap &tm_v, const CUtensorMap &tm_do,
                                              const BwdParams &p, uint8_t *smem_raw) {
    using C = DqCfg<D>;
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    uint8_t *sptr = smem_raw + (sbase - raw_u32);
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * static_cast<uint32_t>(i); };
    auto kslot = [&](int gj) -> uint32_t { return sbase + C::kOffK + static_cast<uint32_t>(gj % C::kKStages) * C::kTile; };
    auto vslot = [&](int gj) -> uint32_t { return sbase + C::kOffV + static_cast<uint32_t>(gj % C::kVStages) * C::kTile; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sptr + C::kOffBar + C::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
    const int BH = p.g.B * p.g.H;
    const int T = BH * p.n_tiles;
    // work unit of rank r: query tile qt (heaviest = the last), slice (b, h); false if empty.
    // ks: the key tiles query tile qt attends (all of [0, reach) without a tile mask);
    // nkv of them, walked in increasing order.
    struct Tile {
        int b, h, qt, start, len, q0, nkv;
        TileSet ks;
    };
    auto tile_at = [&](int r, Tile &t) -> bool {
        const int k = r / BH;
        const int bh = r - k * BH;
        t.qt = p.n_tiles - 1 - k;
        t.b = bh / p.g.H;
        t.h = bh - t.b * p.g.H;
        p.g.slice(t.b, t.start, t.len);
        t.q0 = t.qt * 128;
        if (t.q0 >= t.len) return false;
        const int nkv_all = (t.len + 127) / 128;
        t.ks = row_tiles<SP>(p.g, t.h, t.qt, p.causal ? min(nkv_all, t.qt + 1) : nkv_all);
        t.nkv = t.ks.count();
        return true;
    };

    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i)
            mbar_init(bar(i), (i == C::kBarDPFree || i == C::kBarDSFull || i == C::kBarDSFull + 1 ||
                               i == C::kBarAccFree) ? 256u : 1u);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    int n_k = 0, n_v = 0, n_qt = 0;  // loader: K/V tiles and Q/dO pairs started (for the abort drain)

    if (warp == 8) {
        // ------------------------------------------------------------ loader
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int r = snake_rank(k, cta, G);
                if (r >= T) break;
                Tile t;
                if (!tile_at(r, t) || t.nkv == 0) continue;  // (nkv == 0: the math warps write zeros)
                const int row0 = p.g.tma_row0(t.start), slab = p.g.tma_slab(t.b, t.h);
                // Q_i, dO_i once the previous tile's last S / dP have read theirs
                if (!wait_phase(bar(C::kBarQEmpty), (n_qt & 1) ^ 1, p.ctl, abort_flag)) break;
                if (n_qt != p.ctl.inject_skip_load) {  // (test hook: this tile never arrives)
                    mbar_arrive_expect_tx(bar(C::kBarQFull), 2 * C::kTile);
#pragma unroll
                    for (int x = 0; x < C::kBoxes; ++x) {
                        tma_load_3d(sbase + C::kOffQ + x * 16384, &tm_q, bar(C::kBarQFull), x * 64, row0 + t.q0, slab);
                        tma_load_3d(sbase + C::kOffDO + x * 16384, &tm_do, bar(C::kBarQFull), x * 64, row0 + t.q0,
                                    slab);
                    }
                }
                ++n_qt;
                for (int jt = 0, j = t.ks.next(0); jt < t.nkv; ++jt, j = t.ks.next(j + 1)) {
                    const int gk = n_k, ks = gk % C::kKStages;
                    if (!wait_phase(bar(C::kBarKEmpty + ks), ((gk / C::kKStages) & 1) ^ 1, p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar(C::kBarKFull + ks), C::kTile);
#pragma unroll
                    for (int x = 0; x < C::kBoxes; ++x)
                        tma_load_3d(kslot(gk) + x * 16384, &tm_k, bar(C::kBarKFull + ks), x * 64, row0 + 128 * j,
                                    slab);
                    ++n_k;
                    const int gv = n_v, vs = gv % C::kVStages;
                    if (!wait_phase(bar(C::kBarVEmpty + vs), ((gv / C::kVStages) & 1) ^ 1, p.ctl, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar(C::kBarVFull + vs), C::kTile);
#pragma unroll
                    for (int x = 0; x < C::kBoxes; ++x)
                        tma_load_3d(vslot(gv) + x * 16384, &tm_v, bar(C::kBarVFull + vs), x * 64, row0 + 128 * j,
                                    slab);
                    ++n_v;
                }
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idQ = idesc_bf16_f32(128, D, 0, 1);
            auto issue_s = [&](int gj) {
                const uint32_t ks = kslot(gj);
                const uint32_t col = (gj & 1) ? C::kColS1 : C::kColS0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + col, sw128_desc(sbase + C::kOffQ + kstep_off(kk), 16, 1024),
                           sw128_desc(ks + kstep_off(kk), 16, 1024), idS, kk > 0);
                tc_commit(bar(C::kBarSFull + (gj & 1)));
            };
            auto issue_dp = [&](int gj) {
                const uint32_t vs = vslot(gj);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss(tmem + C::kColDP, sw128_desc(sbase + C::kOffDO + kstep_off(kk), 16, 1024),
                           sw128_desc(vs + kstep_off(kk), 16, 1024), idS, kk > 0);
                tc_commit(bar(C::kBarDPFull));
                tc_commit(bar(C::kBarVEmpty + gj % C::kVStages));  // V_j is free once dP_j is done
            };
            auto wait_k = [&](int gj) {
                return wait_phase(bar(C::kBarKFull + gj % C::kKStages), (gj / C::kKStages) & 1, p.ctl, abort_flag);
            };
            auto wait_v = [&](int gj) {
                return wait_phase(bar(C::kBarVFull + gj % C::kVStages), (gj / C::kVStages) & 1, p.ctl, abort_flag);
            };
            bool ok = true;
            int gbase = 0, n_t = 0;
            for (int k = 0; ok; ++k) {
                const int r = snake_rank(k, cta, G);
                if (r >= T) break;
                Tile t;
                if (!tile_at(r, t) || t.nkv == 0) continue;
                ok = wait_phase(bar(C::kBarQFull), n_t & 1, p.ctl, abort_flag);
                if (ok) ok = wait_k(gbase);
                if (!ok) break;
                tc_fence_after();
                // S buffer gbase & 1 last held dS of step gbase-2, read by a dQ product
                // issued earlier; the dP region was copied out (dP free) before the
                // previous tile's last dQ was issued.
                issue_s(gbase);
                if (n_t > 0) ok = wait_phase(bar(C::kBarDPFree), (gbase - 1) & 1, p.ctl, abort_flag);
                if (ok) ok = wait_v(gbase);
                if (!ok) break;
                tc_fence_after();
                issue_dp(gbase);
                if (t.nkv == 1) tc_commit(bar(C::kBarQEmpty));
                for (int jt = 0; ok && jt < t.nkv; ++jt) {
                    const int gj = gbase + jt;
                    if (jt + 1 < t.nkv) {
                        ok = wait_k(gj + 1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(gj + 1);
                        ok = wait_phase(bar(C::kBarDPFree), gj & 1, p.ctl, abort_flag);
                        if (ok) ok = wait_v(gj + 1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_dp(gj + 1);
                        if (jt + 2 == t.nkv) tc_commit(bar(C::kBarQEmpty));  // last S / dP of the tile
                    }
                    // dQ += dS_j K_j  (A = dS from TMEM: keys 0-63 at columns 0-31, keys 64-127 at 64-95)
                    ok = wait_phase(bar(C::kBarDSFull + (gj & 1)), (gj >> 1) & 1, p.ctl, abort_flag);
                    if (ok && jt == 0 && n_t > 0)  // the previous tile's dQ has been copied out
                        ok = wait_phase(bar(C::kBarAccFree), (n_t - 1) & 1, p.ctl, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t scol = (gj & 1) ? C::kColS1 : C::kColS0;
                    const uint32_t ks = kslot(gj);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t acol = scol + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8);
                        mma_ts(tmem + C::kColDQ, tmem + acol, sw128_desc(ks + kk * 2048, 16384, 1024), idQ,
                               (jt > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(bar(C::kBarKEmpty + gj % C::kKStages));  // K_j is free once dQ_j is done
                }
                if (!ok) break;
                tc_commit(bar(C::kBarDq));
                gbase += t.nkv;
                ++n_t;
            }
            tc_commit(bar(C::kBarDone));
            drain_phase(bar(C::kBarDone), 0, p.ctl, abort_flag);
        }
    } else {
        // ------------------------------------------------------------ P and dS (8 warps)
        // warp w: query rows 32*(w%4).., keys 64*(w/4) .. +63 of each key tile.
        const int q4 = warp & 3, hf = warp >> 2;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const float c2 = p.scale_log2;
        bool ok = true;
        int gbase = 0, n_t = 0;
        for (int k = 0; ok; ++k) {
            const int r = snake_rank(k, cta, G);
            if (r >= T) break;
            Tile t;
            if (!tile_at(r, t)) continue;
            const int qrow = t.q0 + q4 * 32 + lane;  // query row within the slice
            if (t.nkv == 0) {
                // The tile mask leaves query tile qt no key tile: dQ = 0 for its rows
                // (warp w writes columns (w/4)*d/2 ..), and nothing was computed.
                if (qrow < t.len) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.dq + p.g.base(t.b, t.h, t.start, D) +
                                                           static_cast<long long>(qrow) * p.g.row_stride(D) + hf * (D / 2));
#pragma unroll 1
                    for (int v = 0; v < D / 16; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                }
                continue;
            }
            const long long lidx = p.g.base(t.b, t.h, t.start, 1) + static_cast<long long>(qrow) * p.g.row_stride(1);
            const float l2 = (qrow < t.len) ? p.lse2[lidx] : INFINITY;  // rows past the sequence: P = 0
            const float dd = (qrow < t.len) ? p.dvec[lidx] : 0.f;
            const uint8_t *keep = p.g.key_keep ? p.g.key_keep + p.g.keep_base(t.b, t.start) : nullptr;
            for (int jt = 0, j = t.ks.next(0); jt < t.nkv; ++jt, j = t.ks.next(j + 1)) {
                const int gj = gbase + jt;
                // P = 2^(S c - lse2) first: it needs only S, so the exponentials run
                // while the tensor core is still computing dP
                ok = __all_sync(0xffffffffu,
                                wait_phase(bar(C::kBarSFull + (gj & 1)), (gj >> 1) & 1, p.ctl, abort_flag));
                if (!ok) break;
                tc_fence_after();
                const uint32_t scol = (gj & 1) ? C::kColS1 : C::kColS0;
                float pf[64];
                {
                    uint32_t sr[2][32];
#pragma unroll
                    for (int x = 0; x < 2; ++x) tmem_ld32(tmem + lane_off + scol + hf * 64 + x * 32, sr[x]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 64; ++c) pf[c] = ex2_approx(fmaf(__uint_as_float(sr[c >> 5][c & 31]), c2, -l2));
                }
                // masking: keys outside the sequence, above the diagonal, or padded
                const int kb = j * 128 + hf * 64;  // first key of this warp's columns
                int limit = t.len - kb;
                if (p.causal) limit = min(limit, qrow - kb + 1);
                if (limit < 64) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c >= limit) pf[c] = 0.f;
                }
                if (keep != nullptr) {
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        const int c = x * 32 + lane;
                        const uint32_t km = __ballot_sync(0xffffffffu, (c < t.len - kb) && keep[kb + c] != 0);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (!((km >> e) & 1u)) pf[x * 32 + e] = 0.f;
                    }
                }
                // dS = P o (dP - D), written over S as bf16
                ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarDPFull), gj & 1, p.ctl, abort_flag));
                if (!ok) break;
                tc_fence_after();
                uint32_t dr[2][32];
#pragma unroll
                for (int x = 0; x < 2; ++x) tmem_ld32(tmem + lane_off + C::kColDP + hf * 64 + x * 32, dr[x]);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar(C::kBarDPFree));
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 32; c += 2)
                        pk[c >> 1] = pack_bf16x2(pf[x * 32 + c] * (__uint_as_float(dr[x][c]) - dd),
                                                 pf[x * 32 + c + 1] * (__uint_as_float(dr[x][c + 1]) - dd));
                    tmem_st16(tmem + lane_off + scol + hf * 64 + x * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(C::kBarDSFull + (gj & 1)));
            }
            if (!ok) break;
            // ---- epilogue: scale * dQ in bf16 (warp w writes columns (w/4)*d/2 ..)
            ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarDq), n_t & 1, p.ctl, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const bool valid = qrow < t.len;
            __nv_bfloat16 *out = p.dq + p.g.base(t.b, t.h, t.start, D) + static_cast<long long>(qrow) * p.g.row_stride(D);
#pragma unroll 1  // (unrolled, the key loop above runs out of registers)
            for (int c0 = hf * (D / 2); c0 < (hf + 1) * (D / 2); c0 += 32) {
                uint32_t rr[32];
                tmem_ld32(tmem + lane_off + C::kColDQ + c0, rr);
                tmem_wait_ld();
                if (c0 + 32 == (hf + 1) * (D / 2)) {
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarAccFree));
                }
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    pk[c] = pack_bf16x2(__uint_as_float(rr[2 * c]) * p.scale, __uint_as_float(rr[2 * c + 1]) * p.scale);
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
            }
            gbase += t.nkv;
            ++n_t;
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 8 && lane == 0 && *abort_flag) {
        // After an abort, every copy the loader started must land before the CTA exits.
        if (n_qt > 0 && n_qt - 1 != p.ctl.inject_skip_load)
            drain_phase(bar(C::kBarQFull), (n_qt - 1) & 1, p.ctl, abort_flag);
        for (int g = max(0, n_k - C::kKStages); g < n_k; ++g)
            drain_phase(bar(C::kBarKFull + g % C::kKStages), (g / C::kKStages) & 1, p.ctl, abort_flag);
        for (int g = max(0, n_v - C::kVStages); g < n_v; ++g)
            drain_phase(bar(C::kBarVFull + g % C::kVStages), (g / C::kVStages) & 1, p.ctl, abort_flag);
    }
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ============================================================================ kernels
// Persistent: one CTA per SM walks its share of the work units.
template <int D, bool SP>
__global__ void __launch_bounds__(320, 1)
attn_bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_dk_st, const __grid_constant__ CUtensorMap tm_dv_st,
                           const __grid_constant__ BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    dkdv_persistent<D, SP>(tm_q, tm_k, tm_v, tm_do, tm_dk_st, tm_dv_st, p, smem_raw);
}

template <int D, bool SP>
__global__ void __launch_bounds__(320, 1)
attn_bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    dq_persistent<D, SP>(tm_q, tm_k, tm_v, tm_do, p, smem_raw);
}

// ============================================================================ launch
cudaError_t launch_bwd_pre(const BwdLaunch &a, bool zero_dqacc, cudaStream_t stream) {
    const int *cu = a.g.varlen ? a.g.cu_seqlens : nullptr;
    const int D = a.g.d;
    const long long rows_per_cta = (256 / (D / 8)) * kPrePasses;
    const unsigned blocks = static_cast<unsigned>((a.rows_total + rows_per_cta - 1) / rows_per_cta);
    float *z = zero_dqacc ? a.dqacc : nullptr;
    const auto *o = static_cast<const __nv_bfloat16 *>(a.o);
    const auto *dout = static_cast<const __nv_bfloat16 *>(a.dout);
    if (D == 128)
        attn_bwd_pre_kernel<128><<<blocks, 256, 0, stream>>>(o, dout, a.lse, a.dvec, a.lse2, z, a.rows_total, cu,
                                                             a.g.B, a.g.H);
    else
        attn_bwd_pre_kernel<64><<<blocks, 256, 0, stream>>>(o, dout, a.lse, a.dvec, a.lse2, z, a.rows_total, cu,
                                                            a.g.B, a.g.H);
    return cudaGetLastError();
}

template <int D, bool SP>
static cudaError_t launch_bwd_d(const BwdLaunch &a, cudaStream_t stream) {
    BwdParams p{};
    p.g = a.g;
    p.ctl = a.ctl;
    p.dq = static_cast<__nv_bfloat16 *>(a.dq);
    p.dk = static_cast<__nv_bfloat16 *>(a.dk);
    p.dv = static_cast<__nv_bfloat16 *>(a.dv);
    p.dvec = a.dvec;
    p.lse2 = a.lse2;
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    p.causal = a.causal;
    p.n_tiles = (a.g.N + 127) / 128;
    if (a.phases & 1) {
        cudaError_t e = launch_bwd_pre(a, false, stream);
        if (e != cudaSuccess) return e;
    }
    // dK/dV then dQ, as two launches: one grid holding both kinds of CTA measured
    // slower than the two back to back.
    const long long units = static_cast<long long>(a.g.B) * a.g.H * p.n_tiles;
    const dim3 g(static_cast<unsigned>(units < a.num_sms ? units : a.num_sms));
    cudaError_t e;
    if (a.phases & 2) {
        e = cudaFuncSetAttribute(attn_bwd_dkdv_sm100_kernel<D, SP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DkdvCfg<D>::kSmemBytes);
        if (e != cudaSuccess) return e;
        attn_bwd_dkdv_sm100_kernel<D, SP><<<g, 320, DkdvCfg<D>::kSmemBytes, stream>>>(
            a.tm_q, a.tm_k, a.tm_v, a.tm_do, a.tm_dk_st, a.tm_dv_st, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (a.phases & 4) {
        e = cudaFuncSetAttribute(attn_bwd_dq_sm100_kernel<D, SP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DqCfg<D>::kSmemBytes);
        if (e != cudaSuccess) return e;
        attn_bwd_dq_sm100_kernel<D, SP><<<g, 320, DqCfg<D>::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_do, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_bwd(const BwdLaunch &a, cudaStream_t stream) {
    const bool sp = a.g.block_mask != nullptr;
    if (a.g.d == 128) return sp ? launch_bwd_d<128, true>(a, stream) : launch_bwd_d<128, false>(a, stream);
    return sp ? launch_bwd_d<64, true>(a, stream) : launch_bwd_d<64, false>(a, stream);
}

}  // namespace attn
