// attn_bwd_fused_sm100.cu -- single-pass exact-attention backward for B200 (sm_100a).
//
// The backward recomputes the probabilities from Q, K and the forward's logsumexp
// ("4.5 注意力优化实战：从PyTorch到CUDA的完整流程", 第四步 §2: the softmax normaliser
// kept by the forward is reused; dK and dV sweep the query blocks).  With P the
// probabilities, dO the upstream gradient and D_i = sum_c dO_ic O_ic:
//   dV = P^T dO,   dS = P o (dO V^T - D),   dK = scale dS^T Q,   dQ = scale dS K.
//
// One persistent kernel does all five tensor-core products of a (key tile, query
// tile) pair once -- the separate dQ pass of the deterministic backward recomputes
// S and dP, seven products per pair -- and accumulates dQ in fp32 in device memory:
//   work unit = one 128-key tile K_j, V_j of one (b, h), sweeping the 128-row query
//   tiles Q_i, dO_i (from the diagonal when causal):
//     S^T  = K_j Q_i^T            SS, M = 128 keys, N = 128 queries     -> TMEM
//     dP^T = V_j dO_i^T           SS                                    -> TMEM
//     P^T  = 2^(S^T scale log2e - lse2)   written back over S^T as bf16 (math warps)
//     dS   = P o (dP - D)         written to shared memory as bf16, keys x queries
//     dV  += P^T dO_i             TS: A = P^T from TMEM
//     dQ_i = dS K_j               SS: A = dS read query-major (the transposed view
//                                 of the same shared-memory tile), B = K_j
//     dK  += dS^T Q_i             SS: A = dS as stored
//   and four "drain" warps move each dQ_i tile out of TMEM, through a shared-memory
//   staging area of their own, into an fp32 accumulator with TMA reduce-adds (the
//   add happens in L2).  A small kernel first zeroes the accumulator (with the
//   per-row D and lse2 terms) and another one afterwards writes
//   dQ = bf16(scale * accumulator).
// The fp32 additions from different key tiles land in an order that depends on
// scheduling, so dQ may differ between runs in its last bits; the deterministic
// backward (attn_bwd_sm100.cu) avoids that at the price of the two extra products.
//
// Warp roles (512 threads, four warpgroups; registers move by whole warpgroups):
//   warps 0-7   math: warp w owns key rows 32 (w % 4) .. + 31 (its TMEM lane quadrant)
//               and query columns 64 (w / 4) .. + 63 of each pair
//   warps 8-11  dQ drain: warp w reads TMEM lanes 32 (w % 4) .. + 31 = query rows
//   warp 12     TMA loader (K_j, V_j per unit; Q_i, dO_i and the row terms per step)
//   warp 13     TMEM allocator and single-thread tcgen05.mma issuer
//   warps 14-15 idle (they complete the warpgroup that gives registers away)
//
// Tensor memory (512 columns): S^T / P^T [0, 128), dP^T [128, 256), dV, dK after.
// The dQ_i accumulator needs d more columns: at d = 64 it has [384, 448) to itself;
// at d = 128 it takes dP^T's columns once the math warps have read dP^T, and the
// next dP^T is issued only after the drain warps have read dQ_i out.
//
// Shared memory (d = 128): K_j, V_j 32 KB each; Q_i in a two-stage ring with its
// per-row terms; dO_i in one buffer (it is free again once dV_i is done, well
// before dP^T_{i+1} is issued); the dS tile (32 KB); the drain warps' staging area
// (32 KB: two 4 KB boxes per warp, reused as soon as the TMA has read them).
// The next dS is written only after dP^T_{i+1} is complete, which (tensor-core
// operations completing in issue order) implies dQ_i and dK_i, the products that
// read dS, are done.  At a unit's end the loader issues the next unit's loads in the
// order their buffers free up: V_j once the last dP^T is done, the first Q_i and dO_i,
// then K_j once the last dQ is (at d = 64 K_j alternates between two buffers, so it
// need not wait); that unit's K/V tiles and first Q_i, dO_i and row terms have been
// prefetched into L2 meanwhile.
//
// Units are dealt to the CTAs heaviest first in a snake order (SCHED 0), or -- with a
// tile mask, whose units' costs are uneven -- claimed at run time from a global
// counter by the loader, one unit ahead, and published with the unit's query-tile
// bits to the other roles through a shared-memory ring (SCHED 1); when the slices'
// Q, dO and dQ far exceed the L2 cache, the claimed ranks also walk the slices in
// bands that fit it (SCHED 2, rank_to_unit).
//
// Every wait is bounded (see attn_common.cuh); an expired wait stops every role,
// drains the copies in flight and returns with ATTN_ERR_TIMEOUT in the status word.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "attn_common.cuh"
#include "attn_launch.h"

namespace attn {

namespace {

constexpr float kLog2eF = 1.4426950408889634f;

template <int D>
struct FusedCfg {
    static constexpr int kTile = 128 * D * 2;  // K, V, Q or dO tile (bf16)
    static constexpr int kBoxes = D / 64;      // 64-column TMA boxes per tile
    static constexpr int kStages = 2;                      // Q_i ring (and its per-row terms)
    static constexpr int kDoStages = (D == 128) ? 1 : 2;   // dO_i buffers
    static constexpr int kThreads = 512;
    // Launched at 128 registers per thread (the most 512 threads allow); the drain and
    // control warpgroups give registers back, the two math warpgroups take them.
    static constexpr int kLaunchRegs = 128, kRegsMath = 160, kRegsDrain = 96, kRegsCtl = 96;
    static_assert(2 * 128 * kRegsMath + 128 * kRegsDrain + 128 * kRegsCtl <= kThreads * kLaunchRegs,
                  "register reallocation exceeds the launch pool");
    static constexpr int kTmemCols = 512;
    static constexpr int kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
    static constexpr bool kDqOverDp = (D == 128);  // the dQ accumulator reuses dP^T's columns
    static constexpr int kColDQ = kDqOverDp ? kColDP : 256 + 2 * D;
    static_assert(kColDQ + D <= kTmemCols, "tensor memory budget");
    static constexpr int kOffK = 0, kOffV = kTile;
    static constexpr int kOffQ = 2 * kTile;                   // + st * kTile
    static constexpr int kOffDO = kOffQ + kStages * kTile;     // + buffer * kTile
    static constexpr int kOffDS = kOffDO + kDoStages * kTile;  // 128 keys x 128 queries bf16, two 64-query boxes
    static constexpr int kOffStage = kOffDS + 32768;           // + warp * 8192: two {32 x 32} fp32 boxes
    static constexpr int kOffVec = kOffStage + 32768;          // + st * 1024: lse2[128], D[128]
    // K_j buffers: two at d = 64, alternating by unit, so that the next unit's K_j loads
    // while the current unit's last dQ products still read the other (a unit otherwise
    // starts by waiting out that load); at d = 128 shared memory has room for one.
    static constexpr int kKBufs = (D == 64) ? 2 : 1;
    static constexpr int kOffK1 = kOffVec + kStages * 1024;  // the second K_j buffer
    static constexpr int kOffBar = kOffK1 + (kKBufs == 2 ? kTile : 0);
    static constexpr int kBarKFull = 0;
    static constexpr int kBarKEmpty = 1;                       // K_j no longer read (the unit's last dQ done)
    static constexpr int kBarVFull = 2;
    static constexpr int kBarVEmpty = 3;                       // V_j no longer read (the unit's last dP^T done)
    static constexpr int kBarQFull = 4;                        // + st: Q_i landed and its row terms stored (2 arrivals)
    static constexpr int kBarQEmpty = kBarQFull + kStages;     // + st
    static constexpr int kBarDOFull = kBarQEmpty + kStages;    // + buffer
    static constexpr int kBarDOEmpty = kBarDOFull + kDoStages; // + buffer
    static constexpr int kBarSFull = kBarDOEmpty + kDoStages;
    static constexpr int kBarDPFull = kBarSFull + 1;
    static constexpr int kBarPFull = kBarSFull + 2;       // P^T in TMEM (256 math threads)
    static constexpr int kBarDSFull = kBarSFull + 3;      // dS in shared memory, dP^T read (256)
    static constexpr int kBarDQFull = kBarSFull + 4;      // dQ_i product done
    static constexpr int kBarDQFree = kBarSFull + 5;      // dQ_i read out of TMEM (128 drain threads)
    static constexpr int kBarKdv = kBarSFull + 6;         // dV, dK accumulators complete
    static constexpr int kBarAccFree = kBarSFull + 7;     // dV, dK copied out of TMEM (256)
    static constexpr int kBarDone = kBarSFull + 8;
    static constexpr int kBarUFull = kBarSFull + 9;       // + entry: a claimed unit rank is published
    static constexpr int kBarUEmpty = kBarSFull + 13;     // + entry: every role has read it (385)
    static constexpr int kBarKFull1 = kBarSFull + 17;     // the second K_j buffer: loaded / free again
    static constexpr int kBarKEmpty1 = kBarSFull + 18;
    static constexpr int kNumBars = kBarSFull + 17 + (kKBufs == 2 ? 2 : 0);
    // after the barriers: TMEM base, abort flag, 4-entry ring of claimed units
    // ({rank, query-tile bits}, 16 bytes each)
    // debug library, after the ring: a check tag per Q stage and the roles' final counts
    static constexpr int kDebugBytes = kDebugChecks ? 8 * kStages + 32 : 0;
    static constexpr int kSmemUsed = kOffBar + kNumBars * 8 + 80 + kDebugBytes;  // from a 1024-byte-aligned base
    static constexpr int kSmemMax = 232448;
    // The base of dynamic shared memory is expected to be 1024-byte aligned; the
    // kernel checks, and where the slack below cannot cover the misalignment it
    // reports ATTN_ERR_UNSUPPORTED instead of running.
    static constexpr int kSmemBytes = (kSmemUsed + 1024 <= kSmemMax) ? kSmemUsed + 1024 : kSmemMax;
    static_assert(kSmemUsed <= kSmemMax, "exceeds the 227 KB per-CTA shared-memory limit");
    static_assert(kTile % 1024 == 0 && kOffDS % 1024 == 0 && kOffStage % 1024 == 0 && kOffK1 % 1024 == 0,
                  "swizzled tiles must be 1024-byte aligned");
};

struct FusedParams {
    Geom g;
    SyncCtl ctl;
    __nv_bfloat16 *dk, *dv;
    const float *dvec, *lse2;
    float scale;
    float scale_log2;
    int causal;
    int n_tiles;  // 128-row tiles per slice
    int band;     // slices per band of the rank order (rank_to_unit)
    unsigned int *sched;  // claimed deal: {units claimed, CTAs finished} of this launch (else null)
};

__device__ __forceinline__ uint32_t kstep(int kk) { return (kk >> 2) * 16384 + (kk & 3) * 32; }

// One warp's 32 rows x 32 fp32 columns into a staging box laid out as the 128-byte
// swizzle of a {32, 32} fp32 TMA box: row r at r * 128, 16-byte chunk c at
// (c ^ (r % 8)) * 16.  Lane = row.
__device__ __forceinline__ void stage_rows32_f32(uint32_t box, const uint32_t (&r)[32], int lane) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
        st_shared_v4(box + lane * 128 + (((c ^ (lane & 7)) & 7) << 4), r[4 * c], r[4 * c + 1], r[4 * c + 2],
                     r[4 * c + 3]);
}

}  // namespace

// SCHED: how the CTAs get their units.  0: dealt (a snake order over the ranks, unit
// index first over all slices).  1: claimed at run time from a global counter, in rank
// order (tile masks, whose units' costs are uneven).  2: claimed, and the ranks walk
// the slices in bands (rank_to_unit) -- when the slices' Q, dO and dQ far exceed the
// L2 cache.
template <int D, bool SP, int SCHED>
__global__ void __launch_bounds__(512, 1)
attn_bwd_fused_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ CUtensorMap tm_dqacc, const __grid_constant__ FusedParams p) {
    using C = FusedCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    if (sbase - raw_u32 + C::kSmemUsed > static_cast<uint32_t>(C::kSmemBytes)) {  // uniform over the CTA
        if (threadIdx.x == 0) atomicCAS(p.ctl.status, 0, kStatusUnsupported);
        return;
    }
    uint8_t *sptr = smem_raw + (sbase - raw_u32);
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * static_cast<uint32_t>(i); };
    // K_j buffer of the n-th unit with work, its barriers and the phase of its use
    auto kbuf = [](int n) -> int { return C::kKBufs == 2 ? (n & 1) : 0; };
    auto kpar = [](int n) -> uint32_t { return static_cast<uint32_t>(C::kKBufs == 2 ? (n >> 1) & 1 : n & 1); };
    auto koff = [&](int n) -> uint32_t { return sbase + (kbuf(n) ? C::kOffK1 : C::kOffK); };
    auto bar_kfull = [&](int n) -> uint32_t { return bar(kbuf(n) ? C::kBarKFull1 : C::kBarKFull); };
    auto bar_kempty = [&](int n) -> uint32_t { return bar(kbuf(n) ? C::kBarKEmpty1 : C::kBarKEmpty); };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sptr + C::kOffBar + C::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
    const int BH = p.g.B * p.g.H;
    const int T = BH * p.n_tiles;
    // Work unit of rank r (SCHED 0: CTA c takes ranks c, 2G-1-c, 2G+c, ..., a snake
    // order over the units ranked heaviest first; else the ranks it claims, in order,
    // within bands of slices when SCHED = 2): key tile j, slice (b, h); qs = the query
    // tiles that attend key tile j, nq of them, walked in increasing order.
    constexpr bool kDyn = SCHED != 0;
    struct Tile {
        int b, h, j, start, len, kv0, i0, nq;
        TileSet qs;
    };
    // (bits: the unit's query-tile bits as another role read them from the mask)
    auto tile_at = [&](int r, Tile &t, const uint64_t *bits = nullptr) -> bool {
        int bh;
        if constexpr (SCHED == 2) {
            rank_to_unit(r, p.n_tiles, BH, p.band, t.j, bh);
        } else {
            t.j = r / BH;
            bh = r - t.j * BH;
        }
        t.b = bh / p.g.H;
        t.h = bh - t.b * p.g.H;
        p.g.slice(t.b, t.start, t.len);
        t.kv0 = t.j * 128;
        if (t.kv0 >= t.len) return false;
        t.i0 = p.causal ? t.j : 0;
        t.qs = bits ? TileSet{*bits, t.i0, (t.len + 127) / 128, SP} : col_tiles<SP>(p.g, t.h, t.j, t.i0, (t.len + 127) / 128);
        t.nq = t.qs.count();
        return true;
    };
    auto rank_of = [&](int k) { return k * G + ((k & 1) ? (G - 1 - cta) : cta); };
    // Claimed deal: the loader claims each rank, reads the unit's column of the tile
    // mask and publishes {rank, query-tile bits} to the issuer, the drain and the math
    // warps through a 4-entry ring (so only the loader reads the mask); T ends the walk.
    volatile uint64_t *unit_ring = reinterpret_cast<volatile uint64_t *>(tmem_holder + 2);  // 8-byte aligned
    uint64_t unit_bits = 0;  // the query-tile bits of the unit of the role's last rank
    const uint64_t *ubits = kDyn ? &unit_bits : nullptr;
    auto publish_rank = [&](int k, uint64_t &bits) -> int {  // loader, lane 0
        int r = T;
        if (!*abort_flag) r = min(static_cast<int>(atomicAdd(p.sched, 1u)), T);
        bits = 0;
        if (Tile tn; r < T && tile_at(r, tn)) bits = tn.qs.bits;
        if (!wait_phase(bar(C::kBarUEmpty + (k & 3)), ((k >> 2) & 1) ^ 1, p.ctl, abort_flag)) return T;
        unit_ring[2 * (k & 3)] = static_cast<uint64_t>(r);
        unit_ring[2 * (k & 3) + 1] = bits;
        mbar_arrive(bar(C::kBarUFull + (k & 3)));
        return r;
    };
    // Debug library: the loader tags each Q stage fill with {unit rank, query tile, pair
    // number}, which the issuer checks against its own walk when the fill lands; at exit
    // the loader, issuer, math and drain warps must agree on the units and pairs they did.
    uint64_t *const dbg_tag = reinterpret_cast<uint64_t *>(sptr + C::kOffBar + C::kNumBars * 8 + 80);
    uint32_t *const dbg_cnt = reinterpret_cast<uint32_t *>(dbg_tag + C::kStages);
    auto fill_tag = [](int r, int i, int gi) -> uint64_t {
        return (static_cast<uint64_t>(static_cast<uint32_t>(r)) << 32) |
               (static_cast<uint64_t>(static_cast<uint32_t>(i) & 0xFFFFu) << 16) |
               (static_cast<uint32_t>(gi) & 0xFFFFu);
    };
    auto tag_ok = [&](int r, int i, int gi) -> bool {  // issuer, after the fill's full barrier
        if constexpr (kDebugChecks) {
            if (dbg_tag[gi % C::kStages] != fill_tag(r, i, gi)) {
                raise_abort(p.ctl, abort_flag, kStatusDebugCheck);
                return false;
            }
        }
        return true;
    };
    auto consumer_rank = [&](int k) -> int {  // issuer, drain and math threads
        if constexpr (kDyn) {
            if (!wait_phase(bar(C::kBarUFull + (k & 3)), (k >> 2) & 1, p.ctl, abort_flag)) return T;
            const int r = static_cast<int>(unit_ring[2 * (k & 3)]);
            unit_bits = unit_ring[2 * (k & 3) + 1];
            mbar_arrive(bar(C::kBarUEmpty + (k & 3)));
            return r;
        } else {
            return rank_of(k);
        }
    };

    if (warp == 13) {
        tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == C::kBarPFull || i == C::kBarDSFull || i == C::kBarAccFree) cnt = 256;
            if (i == C::kBarDQFree) cnt = 128;
            if (i >= C::kBarQFull && i < C::kBarQFull + C::kStages) cnt = 2;  // the Q copy, then the row terms
            if (i >= C::kBarUEmpty && i < C::kBarUEmpty + 4) cnt = 1 + 128 + 256;  // issuer, drain, math
            mbar_init(bar(i), cnt);
        }
        *abort_flag = 0;
        if constexpr (kDebugChecks)
            for (int i = 0; i < 8; ++i) dbg_cnt[i] = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    int n_q = 0, n_do = 0, n_kv = 0;  // loader: Q, dO and K/V loads started (for the abort drain)
    int n_v = 0, n_k = 0;             // loader: V and K loads started (a unit counts in n_kv once both are)

    if (warp >= 12) {
        setmaxnreg_dec<C::kRegsCtl>();
        if (warp == 12) {
            // ------------------------------------------------------------ loader
            if (lane == 0) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
                tma_prefetch_desc(&tm_do);
            }
            bool ok = true;
            int r_next = 0;  // claimed deal: the next unit, claimed one unit ahead (its L2 prefetch)
            uint64_t bits_next = 0;
            if constexpr (kDyn) {
                if (lane == 0) r_next = publish_rank(0, bits_next);
                r_next = __shfl_sync(0xffffffffu, r_next, 0);
                bits_next = __shfl_sync(0xffffffffu, bits_next, 0);
            }
            for (int k = 0; ok; ++k) {
                int r;
                if constexpr (kDyn) {
                    r = r_next;
                    unit_bits = bits_next;
                    if (r >= T) break;
                    if (lane == 0) r_next = publish_rank(k + 1, bits_next);
                    r_next = __shfl_sync(0xffffffffu, r_next, 0);
                    bits_next = __shfl_sync(0xffffffffu, bits_next, 0);
                } else {
                    r = rank_of(k);
                    if (r >= T) break;
                }
                Tile t;
                if (!tile_at(r, t, ubits) || t.nq == 0) continue;  // (nq == 0: the math warps write zeros)
                const int row0 = p.g.tma_row0(t.start), slab = p.g.tma_slab(t.b, t.h);
                const long long lrow0 = p.g.base(t.b, t.h, t.start, 1), lrs = p.g.row_stride(1);
                // Q_i, dO_i and the row terms of the unit's pair with query tile i
                auto load_pair = [&](int i) -> bool {
                    const int gi = n_q, st = gi % C::kStages;
                    const int q0 = i * 128;
                    // the step's row terms, read before waiting for the stage so that their
                    // global-memory latency overlaps the wait
                    float l2[4], dd[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int q = q0 + u * 32 + lane;
                        l2[u] = INFINITY;  // rows past the sequence: P = 0
                        dd[u] = 0.f;
                        if (q < t.len) {
                            l2[u] = p.lse2[lrow0 + q * lrs];
                            dd[u] = p.dvec[lrow0 + q * lrs];
                        }
                    }
                    if (!__all_sync(0xffffffffu, wait_phase(bar(C::kBarQEmpty + st), ((gi / C::kStages) & 1) ^ 1,
                                                            p.ctl, abort_flag)))
                        return false;
                    // Q_i's copy first, then the row terms once their loads are in: the stage's
                    // full barrier takes both arrivals, so the copy does not wait for them
                    const bool fill = gi != p.ctl.inject_skip_load;  // (test hook: this stage never fills)
                    if (lane == 0 && fill) {
                        if constexpr (kDebugChecks)  // (test hook: one fill's tag written wrong)
                            dbg_tag[st] = fill_tag(r, i, gi) ^ (gi == p.ctl.inject_bad_tag ? 1ull : 0ull);
                        mbar_arrive_expect_tx(bar(C::kBarQFull + st), C::kTile);
#pragma unroll
                        for (int x = 0; x < C::kBoxes; ++x)
                            tma_load_3d(sbase + C::kOffQ + st * C::kTile + x * 16384, &tm_q, bar(C::kBarQFull + st),
                                        x * 64, row0 + q0, slab);
                    }
                    ++n_q;
                    float *vec = reinterpret_cast<float *>(sptr + C::kOffVec + st * 1024);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        vec[u * 32 + lane] = l2[u];
                        vec[128 + u * 32 + lane] = dd[u];
                    }
                    __syncwarp();
                    if (lane == 0 && fill) mbar_arrive(bar(C::kBarQFull + st));
                    // dO_i once dV of the step that last used its buffer is done
                    const int db = gi % C::kDoStages;
                    if (!__all_sync(0xffffffffu, wait_phase(bar(C::kBarDOEmpty + db), ((gi / C::kDoStages) & 1) ^ 1,
                                                            p.ctl, abort_flag)))
                        return false;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar(C::kBarDOFull + db), C::kTile);
#pragma unroll
                        for (int x = 0; x < C::kBoxes; ++x)
                            tma_load_3d(sbase + C::kOffDO + db * C::kTile + x * 16384, &tm_do, bar(C::kBarDOFull + db),
                                        x * 64, row0 + q0, slab);
                    }
                    ++n_do;
                    return true;
                };
                // K_j or V_j once the previous unit has released it
                auto load_kv = [&](int kv) -> bool {
                    const uint32_t full = kv ? bar(C::kBarVFull) : bar_kfull(n_kv);
                    const uint32_t empty = kv ? bar(C::kBarVEmpty) : bar_kempty(n_kv);
                    const uint32_t par = kv ? static_cast<uint32_t>(n_kv & 1) : kpar(n_kv);
                    if (!__all_sync(0xffffffffu, wait_phase(empty, par ^ 1, p.ctl, abort_flag))) return false;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(full, C::kTile);
#pragma unroll
                        for (int x = 0; x < C::kBoxes; ++x)
                            tma_load_3d((kv ? sbase + C::kOffV : koff(n_kv)) + x * 16384, kv ? &tm_v : &tm_k, full,
                                        x * 64, row0 + t.kv0, slab);
                    }
                    if (kv) ++n_v;
                    else ++n_k;
                    return true;
                };
                // In the order the previous unit releases the buffers: V_j after its last dP^T,
                // the first Q_i and dO_i (their stages free up before its last products are
                // done), K_j after its last dQ -- or, with two K_j buffers (free since the unit
                // before), K_j right after V_j, ahead of the first pair's row-term loads.
                const int i_first = t.qs.next(t.i0);
                ok = load_kv(1);
                if (C::kKBufs == 2 && ok) ok = load_kv(0);
                if (ok) ok = load_pair(i_first);
                if (C::kKBufs == 1 && ok) ok = load_kv(0);
                if (!ok) break;
                ++n_kv;
                // the next unit's K and V tiles, and its first Q and dO tiles, into L2 while
                // this unit runs
                auto prefetch_unit = [&](const Tile &t2) {
                    const int r2 = p.g.tma_row0(t2.start), s2 = p.g.tma_slab(t2.b, t2.h);
                    const int q2 = t2.qs.next(t2.i0) * 128;
#pragma unroll
                    for (int x = 0; x < C::kBoxes; ++x) {
                        tma_prefetch_l2_3d(&tm_k, x * 64, r2 + t2.kv0, s2);
                        tma_prefetch_l2_3d(&tm_v, x * 64, r2 + t2.kv0, s2);
                        tma_prefetch_l2_3d(&tm_q, x * 64, r2 + q2, s2);
                        tma_prefetch_l2_3d(&tm_do, x * 64, r2 + q2, s2);
                    }
                    if (!p.g.varlen) {  // and its first row terms (dense: 128 consecutive floats each)
                        const long long b2 = p.g.base(t2.b, t2.h, t2.start, 1) + q2;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            prefetch_l2(p.lse2 + b2 + 32 * c);
                            prefetch_l2(p.dvec + b2 + 32 * c);
                        }
                    }
                };
                if (kDyn && lane == 0) {
                    Tile t2;
                    if (r_next < T && tile_at(r_next, t2, &bits_next) && t2.nq > 0) prefetch_unit(t2);
                }
                if (!kDyn && lane == 0) {
                    for (int k2 = k + 1;; ++k2) {
                        const int r2 = rank_of(k2);
                        if (r2 >= T) break;
                        Tile t2;
                        if (!tile_at(r2, t2) || t2.nq == 0) continue;
                        prefetch_unit(t2);
                        break;
                    }
                }
                for (int it = 1, i = t.qs.next(i_first + 1); it < t.nq; ++it, i = t.qs.next(i + 1)) {
                    ok = load_pair(i);
                    if (!ok) break;
                }
            }
            if (kDebugChecks && lane == 0) {
                dbg_cnt[0] = static_cast<uint32_t>(n_kv);
                dbg_cnt[1] = static_cast<uint32_t>(n_q);
                dbg_cnt[2] = static_cast<uint32_t>(n_do);
            }
        } else if (warp == 13) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
                constexpr uint32_t idKV = idesc_bf16_f32(128, D, 0, 1);   // dV (TS), dK (A = dS as stored)
                constexpr uint32_t idDQ = idesc_bf16_f32(128, D, 1, 1);   // dQ (A = dS read query-major)
                const uint32_t ds = sbase + C::kOffDS;
                // P^T sits in TMEM with queries 0-63 at columns 0-31 and queries 64-127 at
                // columns 64-95 of the S^T region (each math warp writes only inside the
                // columns it read).
                auto acol = [](int kk) -> uint32_t { return kk < 4 ? kk * 8 : 64 + (kk - 4) * 8; };
                uint32_t ks = sbase + C::kOffK;  // the current unit's K_j buffer
                auto issue_s = [&](int gi) {
                    const uint32_t qs = sbase + C::kOffQ + (gi % C::kStages) * C::kTile;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + C::kColS, sw128_desc(ks + kstep(kk), 16, 1024),
                               sw128_desc(qs + kstep(kk), 16, 1024), idS, kk > 0);
                    tc_commit(bar(C::kBarSFull));
                };
                auto issue_dp = [&](int gi) {
                    const uint32_t dos = sbase + C::kOffDO + (gi % C::kDoStages) * C::kTile;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + C::kColDP, sw128_desc(sbase + C::kOffV + kstep(kk), 16, 1024),
                               sw128_desc(dos + kstep(kk), 16, 1024), idS, kk > 0);
                    tc_commit(bar(C::kBarDPFull));
                };
                auto wait_q = [&](int gi) {
                    return wait_phase(bar(C::kBarQFull + gi % C::kStages), (gi / C::kStages) & 1, p.ctl, abort_flag);
                };
                auto wait_do = [&](int gi) {
                    return wait_phase(bar(C::kBarDOFull + gi % C::kDoStages), (gi / C::kDoStages) & 1, p.ctl,
                                      abort_flag);
                };
                bool ok = true;
                int gbase = 0, n_t = 0;
                for (int k = 0; ok; ++k) {
                    const int r = consumer_rank(k);
                    if (r >= T) break;
                    Tile t;
                    if (!tile_at(r, t, ubits) || t.nq == 0) continue;
                    ok = wait_phase(bar_kfull(n_t), kpar(n_t), p.ctl, abort_flag);
                    ks = koff(n_t);
                    if (ok) ok = wait_q(gbase);
                    int dbg_i = t.qs.next(t.i0);  // (debug library: the query tile of pair gi)
                    if (ok) ok = tag_ok(r, dbg_i, gbase);
                    if (!ok) break;
                    tc_fence_after();
                    // S^T's columns are free: the previous unit's last dV, which read P^T from
                    // them, was issued earlier and tensor-core operations complete in order.
                    issue_s(gbase);
                    if (C::kDqOverDp && gbase > 0)  // dP^T's columns held the previous dQ tile
                        ok = wait_phase(bar(C::kBarDQFree), (gbase - 1) & 1, p.ctl, abort_flag);
                    if (ok) ok = wait_phase(bar(C::kBarVFull), n_t & 1, p.ctl, abort_flag);
                    if (ok) ok = wait_do(gbase);
                    if (!ok) break;
                    tc_fence_after();
                    issue_dp(gbase);
                    if (t.nq == 1) tc_commit(bar(C::kBarVEmpty));  // the unit's last dP^T
                    for (int it = 0; ok && it < t.nq; ++it) {
                        const int gi = gbase + it, st = gi % C::kStages;
                        const uint32_t qs = sbase + C::kOffQ + st * C::kTile;
                        const uint32_t dos = sbase + C::kOffDO + (gi % C::kDoStages) * C::kTile;
                        const bool more = it + 1 < t.nq;
                        // dV += P^T dO_i   (K = 128 queries: 8 steps)
                        ok = wait_phase(bar(C::kBarPFull), gi & 1, p.ctl, abort_flag);
                        if (ok && it == 0 && n_t > 0)  // the previous unit's dV / dK have been copied out
                            ok = wait_phase(bar(C::kBarAccFree), (n_t - 1) & 1, p.ctl, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts(tmem + C::kColDV, tmem + C::kColS + acol(kk),
                                   sw128_desc(dos + kk * 2048, 16384, 1024), idKV, (it > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(bar(C::kBarDOEmpty + gi % C::kDoStages));  // dV_i was the last reader of dO_i
                        // S^T_{i+1} may overwrite P^T_i now: dV_i, issued first, completes first
                        // (the math warps keep their P in registers for dS).
                        if (more) {
                            ok = wait_q(gi + 1);
                            if constexpr (kDebugChecks) dbg_i = t.qs.next(dbg_i + 1);
                            if (ok) ok = tag_ok(r, dbg_i, gi + 1);
                            if (!ok) break;
                            tc_fence_after();
                            issue_s(gi + 1);
                        }
                        ok = wait_phase(bar(C::kBarDSFull), gi & 1, p.ctl, abort_flag);
                        if (ok && !C::kDqOverDp && gi > 0)  // the dQ columns held the previous tile
                            ok = wait_phase(bar(C::kBarDQFree), (gi - 1) & 1, p.ctl, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        // dQ_i = dS K_j  (K = 128 keys; A = dS with the queries contiguous, B = K_j
                        // with d contiguous: both read across their 128-byte rows)
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss(tmem + C::kColDQ, sw128_desc(ds + kk * 2048, 16384, 1024),
                                   sw128_desc(ks + kk * 2048, 16384, 1024), idDQ, kk > 0 ? 1u : 0u);
                        tc_commit(bar(C::kBarDQFull));
                        if (!more) tc_commit(bar_kempty(n_t));  // the unit's last reader of K_j
                        // dK += dS^T Q_i  (K = 128 queries; A = dS as stored, keys x queries)
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss(tmem + C::kColDK, sw128_desc(ds + kstep(kk), 16, 1024),
                                   sw128_desc(qs + kk * 2048, 16384, 1024), idKV, (it > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(bar(C::kBarQEmpty + st));  // dK_i was the last reader of Q_i
                        if (more) {
                            if (C::kDqOverDp)  // dP^T_{i+1} overwrites the dQ_i accumulator
                                ok = wait_phase(bar(C::kBarDQFree), gi & 1, p.ctl, abort_flag);
                            if (ok) ok = wait_do(gi + 1);
                            if (!ok) break;
                            tc_fence_after();
                            // (dS_{i+1} is written after this product completes, hence after
                            // dQ_i and dK_i, issued earlier, have read dS_i)
                            issue_dp(gi + 1);
                            if (it + 2 == t.nq) tc_commit(bar(C::kBarVEmpty));  // the unit's last dP^T
                        }
                    }
                    if (!ok) break;
                    tc_commit(bar(C::kBarKdv));
                    gbase += t.nq;
                    ++n_t;
                }
                if constexpr (kDebugChecks) {
                    dbg_cnt[3] = static_cast<uint32_t>(n_t);
                    dbg_cnt[4] = static_cast<uint32_t>(gbase);
                }
                // Every MMA issued above must have finished before TMEM / smem go away.
                tc_commit(bar(C::kBarDone));
                drain_phase(bar(C::kBarDone), 0, p.ctl, abort_flag);
            }
        }
    } else if (warp >= 8) {
        setmaxnreg_dec<C::kRegsDrain>();
        // ---------------------------------------------------------------- dQ drain
        // warp w: query rows 32 (w % 4) .. + 31 of each dQ_i tile, staged 32 columns at a
        // time in two {32 x 32} fp32 boxes of its own; each box is a bulk group of its
        // own, so a box is rewritten as soon as the reduce-add issued two boxes earlier
        // has read it.
        const int q4 = warp & 3;
        const uint32_t tdq = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + C::kColDQ;
        const uint32_t box[2] = {sbase + C::kOffStage + q4 * 8192, sbase + C::kOffStage + q4 * 8192 + 4096};
        auto put = [&](int b, const uint32_t (&r)[32], int col, int row, int slab) {
            if (lane == 0) bulk_wait_read1();  // the group issued before the last one read box b
            __syncwarp();
            stage_rows32_f32(box[b], r, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_reduce_add_3d(&tm_dqacc, box[b], col, row, slab);
                bulk_commit();
            }
        };
        bool ok = true;
        int gbase = 0;
        for (int k = 0; ok; ++k) {
            const int r = consumer_rank(k);
            if (r >= T) break;
            Tile t;
            if (!tile_at(r, t, ubits) || t.nq == 0) continue;
            const int row0 = p.g.tma_row0(t.start) + q4 * 32, slab = p.g.tma_slab(t.b, t.h);
            for (int it = 0, i = t.qs.next(t.i0); it < t.nq; ++it, i = t.qs.next(i + 1)) {
                const int gi = gbase + it;
                const int row = row0 + i * 128;
                ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarDQFull), gi & 1, p.ctl, abort_flag));
                if (!ok) break;
                tc_fence_after();
                uint32_t r0[32], r1[32];
                tmem_ld32(tdq, r0);
                tmem_ld32(tdq + 32, r1);
                tmem_wait_ld();
                if constexpr (!C::kDqOverDp) {
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarDQFree));
                }
                put(0, r0, 0, row, slab);
                put(1, r1, 32, row, slab);
                if constexpr (C::kDqOverDp) {
                    tmem_ld32(tdq + 64, r0);
                    tmem_ld32(tdq + 96, r1);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarDQFree));
                    put(0, r0, 64, row, slab);
                    put(1, r1, 96, row, slab);
                }
            }
            if (!ok) break;
            gbase += t.nq;
        }
        if (kDebugChecks && warp == 8 && lane == 0) dbg_cnt[7] = static_cast<uint32_t>(gbase);
        if (lane == 0) bulk_wait0();  // every reduce-add of this warp has landed
    } else {
        setmaxnreg_inc<C::kRegsMath>();
        // ---------------------------------------------------------------- P^T and dS (warps 0-7)
        // warp w: key rows 32 (w % 4) .., query columns 64 (w / 4) .. + 63 of each query tile.
        const int q4 = warp & 3, hf = warp >> 2;
        const int kr = q4 * 32 + lane;  // key row within the tile
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::kColS + hf * 64;
        const uint32_t tDP = tmem + lane_off + C::kColDP + hf * 64;
        // this thread's row of the dS tile: box hf (queries 64 hf ..), row kr, 128-byte
        // swizzle (chunk c at (c ^ kr % 8) * 16)
        const uint32_t dsrow = sbase + C::kOffDS + hf * 16384 + (kr >> 3) * 1024 + (kr & 7) * 128;
        const float c2 = p.scale_log2;
        bool ok = true;
        int gbase = 0, n_t = 0;
        for (int k = 0; ok; ++k) {
            const int r = consumer_rank(k);
            if (r >= T) break;
            Tile t;
            if (!tile_at(r, t, ubits)) continue;
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
                int lim = p.causal ? key - qb : 0;  // columns c < lim are masked
                if (!kvalid) lim = 64;
                float pf[64];
                const uint64_t c2x2 = f2_pack(c2, c2);
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 l2 = vec[c4];
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {  // column pairs: scale and shift on the f32x2 pipe
                        const int c = c4 * 4 + e;
                        const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[c >> 5][c & 31]),
                                                           __uint_as_float(sr[c >> 5][(c & 31) + 1])),
                                                   c2x2, e ? f2_pack(-l2.z, -l2.w) : f2_pack(-l2.x, -l2.y));
                        float x0, x1;
                        f2_unpack(x2, x0, x1);
                        pf[c] = ex2_approx(x0);
                        pf[c + 1] = ex2_approx(x1);
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
                // dS = P o (dP - D), P taken from registers (fp32), into shared memory
                ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarDPFull), gi & 1, p.ctl, abort_flag));
                if (!ok) break;
                tc_fence_after();
                uint32_t pk[32];
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    uint32_t dr[32];
                    tmem_ld32(tDP + x * 32, dr);
                    tmem_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 dd = vec[32 + x * 8 + c4];
                        const int c = x * 32 + c4 * 4;
                        pk[x * 16 + 2 * c4] = pack_bf16x2(pf[c] * (__uint_as_float(dr[c4 * 4]) - dd.x),
                                                          pf[c + 1] * (__uint_as_float(dr[c4 * 4 + 1]) - dd.y));
                        pk[x * 16 + 2 * c4 + 1] = pack_bf16x2(pf[c + 2] * (__uint_as_float(dr[c4 * 4 + 2]) - dd.z),
                                                              pf[c + 3] * (__uint_as_float(dr[c4 * 4 + 3]) - dd.w));
                    }
                }
                // (dQ_{i-1} and dK_{i-1}, which read the previous dS, are complete: they were
                // issued before dP^T_i, whose completion was just waited for)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(dsrow + (((c ^ (kr & 7)) & 7) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                                 pk[4 * c + 3]);
                fence_proxy_async_smem();  // dS is read by the tensor core (async proxy)
                tc_fence_before();         // and dP^T's columns have been read (dQ_i may overwrite them)
                mbar_arrive(bar(C::kBarDSFull));
            }
            if (!ok) break;
            // ---- epilogue: warps 0-3 write dV, warps 4-7 write scale * dK; TMEM is
            // released (acc free) as soon as the values are in registers
            ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarKdv), n_t & 1, p.ctl, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const bool is_dv = hf == 0;
            __nv_bfloat16 *out = (is_dv ? p.dv : p.dk) + p.g.base(t.b, t.h, t.start, D) +
                                 static_cast<long long>(key) * p.g.row_stride(D);
            const float mul = is_dv ? 1.f : p.scale;
            const uint32_t col = is_dv ? C::kColDV : C::kColDK;
            const bool valid = key < t.len;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t rr[32];
                tmem_ld32(tmem + lane_off + col + c0, rr);
                tmem_wait_ld();
                if (c0 + 32 == D) {
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarAccFree));
                }
                uint32_t o[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    o[c] = pack_bf16x2(__uint_as_float(rr[2 * c]) * mul, __uint_as_float(rr[2 * c + 1]) * mul);
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
                }
            }
            gbase += t.nq;
            ++n_t;
        }
        if (kDebugChecks && warp == 0 && lane == 0) {
            dbg_cnt[5] = static_cast<uint32_t>(n_t);
            dbg_cnt[6] = static_cast<uint32_t>(gbase);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 12 && lane == 0 && *abort_flag) {
        // After an abort, every copy the loader started must land before the CTA exits.
        for (int n = max(0, n_k - C::kKBufs); n < n_k; ++n)  // the last load of each K_j buffer
            drain_phase(bar_kfull(n), kpar(n), p.ctl, abort_flag);
        if (n_v > 0) drain_phase(bar(C::kBarVFull), (n_v - 1) & 1, p.ctl, abort_flag);
        for (int gi = max(0, n_q - C::kStages); gi < n_q; ++gi)
            if (gi != p.ctl.inject_skip_load)
                drain_phase(bar(C::kBarQFull + gi % C::kStages), (gi / C::kStages) & 1, p.ctl, abort_flag);
        for (int gi = max(0, n_do - C::kDoStages); gi < n_do; ++gi)
            drain_phase(bar(C::kBarDOFull + gi % C::kDoStages), (gi / C::kDoStages) & 1, p.ctl, abort_flag);
    }
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if constexpr (kDebugChecks) {
        // without an abort, every role walked the same units and pairs
        if (threadIdx.x == 0 && !*abort_flag) {
            const uint32_t *c = dbg_cnt;
            const bool agree = c[0] == c[3] && c[3] == c[5] && c[1] == c[4] && c[2] == c[4] && c[4] == c[6] &&
                               c[4] == c[7];
            if (!agree) atomicCAS(p.ctl.status, 0, kStatusDebugCheck);
        }
    }
    if constexpr (kDyn) {
        // the last CTA to finish returns the counters to zero for the pair's next launch
        if (threadIdx.x == 0) {
            __threadfence();
            if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
                atomicExch(p.sched, 0u);
                atomicExch(p.sched + 1, 0u);
            }
        }
    }
}

// dQ = bf16(scale * accumulator) over the rows that hold tokens (the flat [rows, d]
// order of q's layout); 8 elements per thread and iteration.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float *__restrict__ acc,
                                                                  __nv_bfloat16 *__restrict__ dq, long long rows,
                                                                  float scale, const int32_t *cu_seqlens, int nseq,
                                                                  int H) {
    long long limit = rows;
    if (cu_seqlens) limit = min(rows, static_cast<long long>(cu_seqlens[nseq]) * H);
    const long long n8 = limit * (D / 8);
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    const float4 *a4 = reinterpret_cast<const float4 *>(acc);
    uint4 *d4 = reinterpret_cast<uint4 *>(dq);
    auto cvt = [&](const float4 &a, const float4 &b) {
        return make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                          pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
    };
    // two groups of 8 per iteration, their four 16-byte loads issued first (read once:
    // streaming loads that L2 may evict first)
    long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + stride < n8; i += 2 * stride) {
        const float4 a0 = __ldcs(a4 + 2 * i), b0 = __ldcs(a4 + 2 * i + 1);
        const float4 a1 = __ldcs(a4 + 2 * (i + stride)), b1 = __ldcs(a4 + 2 * (i + stride) + 1);
        d4[i] = cvt(a0, b0);
        d4[i + stride] = cvt(a1, b1);
    }
    if (i < n8) d4[i] = cvt(__ldcs(a4 + 2 * i), __ldcs(a4 + 2 * i + 1));
}

template <int D, bool SP, int SCHED>
static cudaError_t launch_fused_kernel(const BwdLaunch &a, const FusedParams &p, cudaStream_t stream) {
    using C = FusedCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_fused_sm100_kernel<D, SP, SCHED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // The in-kernel register reallocation assumes the launch register count it was
    // sized for; with fewer, an increase could never be satisfied, so refuse.
    static const cudaError_t regs_ok = [] {
        cudaFuncAttributes fa{};
        const cudaError_t r = cudaFuncGetAttributes(&fa, attn_bwd_fused_sm100_kernel<D, SP, SCHED>);
        if (r != cudaSuccess) return r;
        return fa.numRegs == C::kLaunchRegs ? cudaSuccess : cudaErrorInvalidKernelImage;
    }();
    if (regs_ok != cudaSuccess) return regs_ok;
    const long long units = static_cast<long long>(a.g.B) * a.g.H * p.n_tiles;
    const dim3 grid(static_cast<unsigned>(units < a.num_sms ? units : a.num_sms));
    attn_bwd_fused_sm100_kernel<D, SP, SCHED><<<grid, C::kThreads, C::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v,
                                                                                             a.tm_do, a.tm_dqacc, p);
    return cudaGetLastError();
}

template <int D, bool SP>
static cudaError_t launch_fused_d(const BwdLaunch &a, cudaStream_t stream) {
    using C = FusedCfg<D>;
    cudaError_t e;
    if (a.phases & 8) {
        if ((e = launch_bwd_pre(a, true, stream)) != cudaSuccess) return e;
    }
    if (a.phases & 16) {
        FusedParams p{};
        p.g = a.g;
        p.ctl = a.ctl;
        p.dk = static_cast<__nv_bfloat16 *>(a.dk);
        p.dv = static_cast<__nv_bfloat16 *>(a.dv);
        p.dvec = a.dvec;
        p.lse2 = a.lse2;
        p.scale = a.scale;
        p.scale_log2 = a.scale * kLog2eF;
        p.causal = a.causal;
        p.n_tiles = (a.g.N + 127) / 128;
        // per slice the pairs stream Q, dO (bf16), the fp32 dQ accumulator and the row terms
        p.band = l2_band(a.g.B * a.g.H, static_cast<double>(a.g.N) * (8.0 * a.g.d + 8.0));
        if (forced_band() > 0) p.band = min(forced_band(), a.g.B * a.g.H);  // (test hook)
        // tile masks: claimed units; banded rank order: claimed too (the static deal of a
        // banded order balances badly); otherwise dealt
        p.sched = nullptr;
        const bool banded = p.band < a.g.B * a.g.H;
        if (SP || banded) {
            p.sched = next_sched_slot();
            if (p.sched == nullptr) return cudaErrorInvalidSymbol;
        }
        if (banded) e = launch_fused_kernel<D, SP, 2>(a, p, stream);
        else if constexpr (SP) e = launch_fused_kernel<D, SP, 1>(a, p, stream);
        else e = launch_fused_kernel<D, SP, 0>(a, p, stream);
        if (e != cudaSuccess) return e;
    }
    if (a.phases & 32) {
        const long long n8 = a.rows_total * (D / 8);
        const long long want = (n8 + 255) / 256;
        const unsigned blocks = static_cast<unsigned>(want < 148LL * 16 ? (want > 0 ? want : 1) : 148LL * 16);
        attn_bwd_dq_convert_kernel<D><<<blocks, 256, 0, stream>>>(a.dqacc, static_cast<__nv_bfloat16 *>(a.dq),
                                                                  a.rows_total, a.scale,
                                                                  a.g.varlen ? a.g.cu_seqlens : nullptr, a.g.B, a.g.H);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_bwd_fused(const BwdLaunch &a, cudaStream_t stream) {
    const bool sp = a.g.block_mask != nullptr;
    if (a.g.d == 128) return sp ? launch_fused_d<128, true>(a, stream) : launch_fused_d<128, false>(a, stream);
    return sp ? launch_fused_d<64, true>(a, stream) : launch_fused_d<64, false>(a, stream);
}

}  // namespace attn
