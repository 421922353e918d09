// attn_fwd_sm100.cu -- fused exact-attention forward for B200 (sm_100a).
//
// A work unit is 256 query rows of one (sequence, head) slice, as two 128-row
// tiles Q0 and Q1, which sweeps the key/value tiles of 128 keys with the online
// softmax recurrence ("4.5 注意力优化实战：从PyTorch到CUDA的完整流程", 第三步 §1;
// codechina FlashAttention article §3.2): per query row a running max m, a running
// sum l and an un-normalised output accumulator, rescaled when m moves, divided by
// l at the end.  The 128 x 128 score tile lives only in tensor memory.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for Q0 (warp w owns TMEM lanes 32*(w%4)..+31, one row/thread)
//   warps 4-7  softmax for Q1
//   warp  8    TMA producer: Q0/Q1 once, then K_j, V_j into a ring of shared-memory
//              slots guarded by full/empty mbarriers (the pages' double buffering,
//              done by the copy engine instead of the SMs)
//   warp  9    TMEM allocator and single-thread tcgen05.mma issuer
//   warps 10-11 idle: with warps 8-9 they form the warpgroup that hands registers
//              to the two softmax warpgroups (setmaxnreg)
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   S0 = cols [0,128)  S1 = [128,256)   fp32 scores Q_t K_j^T;
//   P_t (bf16, packed 2 per column) overwrites the first 64 columns of S_t;
//   O0 = [256, 256+d)  O1 = [256+d, 256+2d)   fp32 output accumulators.
//
// MMA issue order per key tile j (single thread, in order):
//   PV0(j) [O0 += P0 V_j], S0(j+1), PV1(j), S1(j+1)
// so the tensor core computes tile 1's product while the Q0 softmax warps work
// on S0(j+1) and vice versa.  Because tcgen05 operations issued by one thread
// complete in order, the commit that publishes S_t(j+1) also proves PV_t(j) is
// done, which is what makes reading/rescaling O_t and overwriting P_t safe.
//
// The kernel is persistent: one CTA per SM walks its units, ranked heaviest
// first (causal: the last query rows see the most keys) and dealt to the CTAs in
// a snake order.  Every barrier counts phases across units and the key/value ring
// runs on, so the next unit's Q tiles load as soon as the current unit's last
// S products are done and its first S products overlap the current epilogue.
// With a tile mask or packed sequences (units of uneven cost) the CTAs instead
// claim the units at run time (DYN: a global counter; the producer publishes each
// claimed unit to the other roles through a small shared-memory ring), in bands of
// slices whose K/V fit the L2 cache when all of it would not (rank_to_unit).  At
// d = 64, causal Q1's extra diagonal key tile is swept first, so that both tiles
// end a unit on the same step (FwdUnit::ufirst).
//
// Exponentials are base 2: p = 2^(s * scale * log2(e) - m).  The running max is
// only moved when a row's new max exceeds the one in use by more than 8 (log2
// units), so O is rescaled rarely (lazy correction); O, l and lse always refer to
// the same m, which keeps the final O / l and lse = (m + log2 l) ln 2 exact.
// A row that sees no key keeps m = -inf and l = 0 and writes O = 0, lse = -inf
// (the _safe_softmax rule of "Profiling in PyTorch (part 3)", math backend).
//
// With a tile mask (block-sparse) the kernel runs with one query tile per CTA and two
// CTAs per SM (NT = 1; 256 threads: softmax warps 0-3, producer warp 4, issuer warp 5,
// 256 TMEM columns: S0 = [0,128), O0 = [128, 128+d)): each CTA sweeps only the key
// tiles its own tile attends, with a K/V ring of its own, so a tile never waits for
// the other tile of a pair (whose key tiles differ) and one CTA's unit change
// overlaps the other CTA's work.
//
// With e4m3 operands (F8, the FP8 direction of the codechina article's §9) both
// products are kind::f8f6f4 with fp32 accumulation; P is rounded to e4m3 and
// written to a swizzled shared-memory tile (the A operand of P V) instead of TMEM,
// and V is read as it is stored, as the MN-major B operand.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "attn_common.cuh"
#include "attn_launch.h"

namespace attn {

// F8: Q, K and V in e4m3 (V, keys x d, is the MN-major B operand of P V as in the
// bf16 path), P rounded to e4m3 in shared memory, fp32 accumulation.
// NT: 128-row query tiles per CTA.  NT = 2: one CTA per SM, its two tiles share every
// K/V tile and take turns on the tensor core.  NT = 1 (tile masks, where the query
// tiles of a pair attend different key tiles): two CTAs per SM, each sweeping the key
// tiles of its own query tile with a ring of its own, so neither waits for the other
// at the end of a unit and neither loads a K/V tile for the other.
template <int D, bool F8 = false, int NT = 2>
struct FwdCfg {
    static constexpr int kEsz = F8 ? 1 : 2;                // bytes per Q/K/V element
    static constexpr int kTileBytes = 128 * D * kEsz;      // one 128-row tile
    // swizzled boxes per tile: 64-column bf16 boxes (128-byte swizzle); one e4m3 box of
    // d bytes per row (128-byte swizzle at d = 128, 64-byte swizzle at d = 64)
    static constexpr int kBoxes = F8 ? 1 : D / 64;
    static constexpr int kKSteps = D * kEsz / 32;          // 32-byte K steps of S = Q K^T
    static_assert(NT == 1 || NT == 2, "one or two query tiles per CTA");
    // K/V ring: at NT = 1 what half an SM's shared memory leaves after Q, P (e4m3) and
    // the output stage
    static constexpr int kStages = NT == 1 ? (F8 ? (D == 128 ? 4 : 8) : (D == 128 ? 2 : 5))
                                           : F8 ? (D == 128 ? 8 : 16) : (D == 128) ? 4 : 8;
    // NT + 1 warpgroups: NT softmax groups, and one with the TMA producer, the MMA
    // issuer and two idle warps (registers move by whole warpgroups).  Launched at the
    // most registers per thread the CTAs of one SM allow (NT = 2: 384 threads, 168;
    // NT = 1: two CTAs of 256, 128), the control group gives registers back and the
    // softmax groups take them: 2*128*200 + 128*104 = 384*168; at NT = 1
    // 128*184 + 128*72 (d = 128) or 128*200 + 128*56 (d = 64) = 256*128, the faster
    // split of each (same-box timings).
    static constexpr int kThreads = 128 * (NT + 1);
    static constexpr int kCtasPerSm = NT == 1 ? 2 : 1;
    static constexpr int kLaunchRegs = NT == 1 ? 128 : 168;
    static constexpr int kRegsSoftmax = (NT == 1 && D == 128) ? 184 : 200;
    static constexpr int kRegsControl = NT == 1 ? 256 - kRegsSoftmax : 104;
    static_assert(NT * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kLaunchRegs,
                  "register reallocation exceeds the launch pool");
    static constexpr int kProducerWarp = 4 * NT, kIssuerWarp = 4 * NT + 1;
    static constexpr int kTmemCols = NT == 1 ? 256 : 512;
    // column pairs c (of each 32-pair half row) whose exponentials come from the FMA
    // pipe: bit (c % 8) set.  Measured best: one pair in eight with e4m3 operands and
    // with bf16 at d = 64 (where the exponentials outweigh the products), none at
    // bf16 d = 128.
    static constexpr uint32_t kPolyPairs = (F8 || D == 64) ? 0x80u : 0u;
    static constexpr int kColS0 = 0, kColS1 = 128, kColO0 = 128 * NT, kColO1 = 128 * NT + D;
    // barrier indices
    static constexpr int kBarQ = 0;
    static constexpr int kBarFull = 1;                       // + slot
    static constexpr int kBarEmpty = 1 + kStages;            // + slot
    static constexpr int kBarS = 1 + 2 * kStages;            // + tile
    static constexpr int kBarP = 3 + 2 * kStages;            // + tile
    static constexpr int kBarO = 5 + 2 * kStages;            // + tile
    static constexpr int kBarDone = 7 + 2 * kStages;
    static constexpr int kBarQEmpty = 8 + 2 * kStages;       // the unit's last S products are done
    static constexpr int kBarUFull = 9 + 2 * kStages;        // + entry: a claimed unit rank is published
    static constexpr int kBarUEmpty = 13 + 2 * kStages;      // + entry: every role has read it
    static constexpr int kNumBars = 17 + 2 * kStages;
    static constexpr int kSmemTiles = (NT + kStages) * kTileBytes;
    static constexpr int kOffP = kSmemTiles;                   // e4m3 P_t: 128 x 128 bytes per tile
    static constexpr int kOffStage = kOffP + (F8 ? NT * 16384 : 0);  // 2 KB output stage per softmax warp
    static constexpr int kOffBar = kOffStage + 4 * NT * 2048;
    // after the barriers: TMEM base, abort flag, 4-entry ring of claimed units
    // ({rank, key-tile bits}, 16 bytes each)
    // debug library, after the ring: a check tag per K/V slot and the roles' final counts
    static constexpr int kDebugBytes = kDebugChecks ? 8 * kStages + 32 : 0;
    static constexpr int kSmemBytes = 1024 + kOffBar + kNumBars * 8 + 96 + kDebugBytes;
    static_assert(kTileBytes % 1024 == 0, "swizzled shared-memory tiles must be 1024-byte aligned");
    // 227 KB per CTA; two CTAs share an SM's 228 KB less 1 KB reserved per CTA
    static_assert(kSmemBytes <= (NT == 1 ? 115712 : 232448), "exceeds the per-CTA shared-memory limit");
};

struct FwdParams {
    Geom g;
    SyncCtl ctl;
    __nv_bfloat16 *o;
    float *lse;
    float scale_log2;  // scale * log2(e) (e4m3: times the Q and K dequantisation scales)
    float o_scale;     // 1, or the V dequantisation scale (e4m3)
    int causal;
    int n_units;       // (128 NT)-row query blocks per slice
    int band;          // slices per band of the rank order (rank_to_unit; DYN only)
    unsigned int *sched;  // dynamic deal: {units claimed, CTAs finished} of this launch (else null)
};

// Unit r of the persistent schedule: k = r / (B*H) counts down the (128 NT)-row
// blocks from the last one, so ranks are ordered heaviest first for causal masking.
// CTA c of G takes ranks c, 2G-1-c, 2G+c, 4G-1-c, ... (snake order), or, with a
// tile mask (whose rows make the units' costs uneven), the next unclaimed rank each
// time it starts a unit (a global counter: the CTAs that draw light units draw more).
struct FwdUnit {
    int b, h, start, len, m0;
    int nkv0, nkv1;  // key tiles in reach of Q0 and Q1 (0: the tile lies past the sequence or NT = 1)
    TileSet ts0, ts1;  // the key tiles Q0 / Q1 actually attend (all of them without a tile mask)
    __device__ __forceinline__ int nkv(int t) const { return t ? nkv1 : nkv0; }
    __device__ __forceinline__ int nkv_max() const { return max(nkv0, nkv1); }
    __device__ __forceinline__ bool live(int t, int j) const { return t ? ts1.has(j) : ts0.has(j); }
    // first key tile >= x that either tile attends (nkv_max() if none): the key/value
    // tiles the unit loads.  A set with no member >= x returns its own end, which
    // must not win the minimum.
    __device__ __forceinline__ int unext(int x) const {
        const int a = ts0.next(x), b = ts1.next(x);
        const int r = min(a < ts0.hi ? a : INT_MAX, b < ts1.hi ? b : INT_MAX);
        return r == INT_MAX ? nkv_max() : r;
    }
    // Sweep order.  Causal, without a tile mask, Q1 reaches one key tile past Q0 (its
    // diagonal tile): that tile goes first, then the shared tiles in increasing order,
    // so that both tiles finish a unit on the same step -- the step Q1 runs alone falls
    // at the start of the next unit, where Q0's warps spend it writing the previous
    // unit's output, instead of at the end, where both would wait.  (The online
    // softmax does not depend on the order of the key tiles.)
    // (Used at d = 64, where a unit is short; at d = 128 the extra code cost more than the
    // idle step, measured.)
    bool diag_first;
    template <bool DF>
    __device__ __forceinline__ int ufirst() const { return (DF && diag_first) ? nkv1 - 1 : unext(0); }
    template <bool DF>
    __device__ __forceinline__ int uafter(int j) const {  // the unit's key tile after j (nkv_max(): none)
        if (!(DF && diag_first)) return unext(j + 1);
        if (j == nkv1 - 1) return nkv1 > 1 ? 0 : nkv1;
        return j + 1 < nkv1 - 1 ? j + 1 : nkv1;
    }
    template <bool DF>
    __device__ __forceinline__ int ulast(int t) const {  // Q_t's last key tile in sweep order
        return (t == 1 && DF && diag_first) ? (nkv1 > 1 ? nkv1 - 2 : 0) : (t ? ts1.last() : ts0.last());
    }
};

// The unit of rank r.  Sets: also build the tile sets (the epilogue needs only the
// unit's position), from the mask or, if `bits` is given, from Q0's key-tile bits
// read by another role (one query tile per CTA, or no mask).  BANDED: ranks walk
// bands of slices (rank_to_unit).
template <bool SP, int NT, bool BANDED, bool Sets = true>
__device__ __forceinline__ bool fwd_unit(const FwdParams &p, int r, FwdUnit &u, const uint64_t *bits = nullptr) {
    const int BH = p.g.B * p.g.H;
    int kk, bh;
    if constexpr (BANDED) {
        rank_to_unit(r, p.n_units, BH, p.band, kk, bh);
    } else {
        kk = r / BH;
        bh = r - kk * BH;
    }
    u.b = bh / p.g.H;
    u.h = bh - u.b * p.g.H;
    p.g.slice(u.b, u.start, u.len);
    u.m0 = (p.n_units - 1 - kk) * 128 * NT;
    if (u.m0 >= u.len) return false;
    const int nkv_all = (u.len + 127) / 128;
    const int r1 = u.m0 + 128;
    u.nkv0 = p.causal ? min(nkv_all, u.m0 / 128 + 1) : nkv_all;
    u.nkv1 = (NT == 1 || r1 >= u.len) ? 0 : (p.causal ? min(nkv_all, r1 / 128 + 1) : nkv_all);
    u.diag_first = !SP && p.causal && u.nkv1 == u.nkv0 + 1;
    if constexpr (Sets) {
        if (bits != nullptr) {
            u.ts0 = TileSet{*bits, 0, u.nkv0, SP};
            u.ts1 = TileSet{0ull, 0, u.nkv1, SP};
        } else {
            u.ts0 = row_tiles<SP>(p.g, u.h, u.m0 / 128, u.nkv0);
            u.ts1 = row_tiles<SP>(p.g, u.h, u.m0 / 128 + 1, u.nkv1);
        }
    }
    return true;
}

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

// SP: a tile mask (block-sparse attention) is given.  F8: e4m3 inputs.  NT: query
// tiles per CTA (see FwdCfg).  DYN: units are claimed at run time (a global counter)
// instead of dealt, in rank order over bands of slices (rank_to_unit): tile masks and
// packed sequences, whose units' costs are uneven.
template <int D, bool SP, bool F8, int NT, bool DYN>
__global__ void __launch_bounds__(FwdCfg<D, F8, NT>::kThreads, FwdCfg<D, F8, NT>::kCtasPerSm)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o_st,
                      const __grid_constant__ FwdParams p) {
    using C = FwdCfg<D, F8, NT>;
    static_assert(!(SP && DYN && NT == 2), "a run-time claim publishes the key-tile bits of one tile");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    uint8_t *sptr = smem_raw + (sbase - raw_u32);
    const uint32_t bars = sbase + C::kOffBar;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    auto slot = [&](int s) -> uint32_t { return sbase + static_cast<uint32_t>(NT + s) * C::kTileBytes; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sptr + C::kOffBar + C::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
    const int n_ranks = p.g.B * p.g.H * p.n_units;
    // Dynamic deal: the producer claims each unit rank, reads the unit's mask row and
    // publishes {rank, Q0's key-tile bits} to the other roles through a 4-entry ring (so
    // only the producer reads the mask); n_ranks ends the walk.
    constexpr bool kDyn = DYN;
    constexpr bool kDiagFirst = D == 64;  // see FwdUnit::ufirst
    volatile uint64_t *unit_ring = reinterpret_cast<volatile uint64_t *>(tmem_holder + 2);  // 8-byte aligned
    uint64_t unit_bits = 0;  // key-tile bits of the unit of the role's last rank (dynamic deal)
    auto claim_rank = [&](int k) -> int {  // producer
        int r = n_ranks;
        if (!*abort_flag) r = min(static_cast<int>(atomicAdd(p.sched, 1u)), n_ranks);
        unit_bits = 0;
        if (FwdUnit un; r < n_ranks && fwd_unit<SP, NT, DYN>(p, r, un)) unit_bits = un.ts0.bits;
        if (!wait_phase(bar(C::kBarUEmpty + (k & 3)), ((k >> 2) & 1) ^ 1, p.ctl, abort_flag)) return n_ranks;
        unit_ring[2 * (k & 3)] = static_cast<uint64_t>(r);
        unit_ring[2 * (k & 3) + 1] = unit_bits;
        mbar_arrive(bar(C::kBarUFull + (k & 3)));
        return r;
    };
    auto take_rank = [&](int k) -> int {  // issuer and softmax threads
        if (!wait_phase(bar(C::kBarUFull + (k & 3)), (k >> 2) & 1, p.ctl, abort_flag)) return n_ranks;
        const int r = static_cast<int>(unit_ring[2 * (k & 3)]);
        unit_bits = unit_ring[2 * (k & 3) + 1];
        mbar_arrive(bar(C::kBarUEmpty + (k & 3)));
        return r;
    };
    auto static_rank = [&](int k) -> int { return k * G + ((k & 1) ? (G - 1 - cta) : cta); };
    // Debug library: the producer tags each ring fill with {unit rank, key tile, fill
    // number}, which the issuer checks against its own walk when the fill lands; at exit
    // the roles' counts (units, fills, S phases per tile) must agree.
    uint64_t *const dbg_tag = reinterpret_cast<uint64_t *>(sptr + C::kOffBar + C::kNumBars * 8 + 96);
    uint32_t *const dbg_cnt = reinterpret_cast<uint32_t *>(dbg_tag + C::kStages);
    auto fill_tag = [](int r, int j, int fill) -> uint64_t {
        return (static_cast<uint64_t>(static_cast<uint32_t>(r)) << 32) |
               (static_cast<uint64_t>(static_cast<uint32_t>(j) & 0xFFFFu) << 16) |
               (static_cast<uint32_t>(fill) & 0xFFFFu);
    };
    auto tag_ok = [&](int r, int fill, int j) -> bool {  // issuer, after the fill's full barrier
        if constexpr (kDebugChecks) {
            if (dbg_tag[fill % C::kStages] != fill_tag(r, j, fill)) {
                raise_abort(p.ctl, abort_flag, kStatusDebugCheck);
                return false;
            }
        }
        return true;
    };
    // walks this CTA's units in order (RANK(k): the role's way to get its k-th rank;
    // the static deal's last round can hold ranks past the end); every role sees the
    // same ranks
#define FOR_EACH_UNIT(u, RANK)                                   \
    for (int k_ = 0; kDyn || k_ * G < n_ranks; ++k_)             \
        if (const int r_ = (RANK)(k_); kDyn && r_ >= n_ranks)    \
            break;                                               \
        else if (FwdUnit u; r_ < n_ranks && fwd_unit<SP, NT, DYN>(p, r_, u, kDyn ? &unit_bits : nullptr))
    auto producer_rank = [&](int k) -> int {
        if constexpr (kDyn) return claim_rank(k);
        else return static_rank(k);
    };
    auto consumer_rank = [&](int k) -> int {
        if constexpr (kDyn) return take_rank(k);
        else return static_rank(k);
    };

    if (warp == C::kIssuerWarp) {
        tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == C::kBarP || i == C::kBarP + 1) cnt = 128;
            if (i >= C::kBarUEmpty && i < C::kBarUEmpty + 4) cnt = 1 + 128 * NT;  // issuer + softmax threads
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
    int n_issued = 0;  // producer: ring loads 0 .. n_issued-1 were started (except a skipped one)
    int n_qload = 0;   // producer: Q pairs whose load was started
    if (warp >= 4 * NT) {
    setmaxnreg_dec<C::kRegsControl>();
    if (warp == C::kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            bool ok = true;
            int idx = 0;  // ring position, continuing across units
            FOR_EACH_UNIT(u, producer_rank) {
                if (!ok) break;
                const int nkv_max = u.nkv_max();
                if (u.unext(0) >= nkv_max) continue;  // no tile pair to compute (tile mask)
                const int row0 = p.g.tma_row0(u.start), slab = p.g.tma_slab(u.b, u.h);
                // the unit's Q tiles once the previous unit's last S products have read theirs
                if (!wait_phase(bar(C::kBarQEmpty), (n_qload & 1) ^ 1, p.ctl, abort_flag)) break;
                mbar_arrive_expect_tx(bar(C::kBarQ), NT * C::kTileBytes);
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int x = 0; x < C::kBoxes; ++x)
                        tma_load_3d(sbase + t * C::kTileBytes + x * 16384, &tm_q, bar(C::kBarQ), x * (128 / C::kEsz),
                                    row0 + u.m0 + 128 * t, slab);
                ++n_qload;
                // the key-padding flags of the unit (if any) are brought into L1 with the
                // K/V tiles, so that the softmax warps' reads of them hit L1
                const uint8_t *keep = p.g.key_keep ? p.g.key_keep + p.g.keep_base(u.b, u.start) : nullptr;
                // the key tiles either query tile attends (with a tile mask, NT = 1: those of
                // the CTA's one tile)
                for (int j = u.ufirst<kDiagFirst>(); j < nkv_max && ok; j = u.uafter<kDiagFirst>(j)) {
                    if (keep != nullptr) {
                        prefetch_l1(keep + 128 * j);
                        prefetch_l1(keep + 128 * j + 127);
                    }
#pragma unroll
                    for (int kv = 0; kv < 2; ++kv, ++idx) {
                        const int s = idx % C::kStages;
                        if (!wait_phase(bar(C::kBarEmpty + s), ((idx / C::kStages) & 1) ^ 1, p.ctl, abort_flag)) {
                            ok = false;
                            break;
                        }
                        if (idx == p.ctl.inject_skip_load) continue;  // test hook: this slot never fills
                        if constexpr (kDebugChecks)  // (test hook: one fill's tag written wrong)
                            dbg_tag[s] = fill_tag(r_, j, idx) ^ (idx == p.ctl.inject_bad_tag ? 1ull : 0ull);
                        mbar_arrive_expect_tx(bar(C::kBarFull + s), C::kTileBytes);
#pragma unroll
                        for (int x = 0; x < C::kBoxes; ++x)
                            tma_load_3d(slot(s) + x * 16384, kv ? &tm_v : &tm_k, bar(C::kBarFull + s),
                                        x * (128 / C::kEsz), row0 + 128 * j, slab);
                        n_issued = idx + 1;
                    }
                }
            }
            if constexpr (kDebugChecks) {
                dbg_cnt[0] = static_cast<uint32_t>(n_qload);
                dbg_cnt[1] = static_cast<uint32_t>(idx);
            }
        }
    } else if (warp == C::kIssuerWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = F8 ? idesc_e4m3_f32(128, 128, 0) : idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idPV = F8 ? idesc_e4m3_f32(128, D, 1) : idesc_bf16_f32(128, D, 0, 1);
            const uint32_t colS[2] = {C::kColS0, C::kColS1};
            const uint32_t colO[2] = {C::kColO0, C::kColO1};
            // K-major operand descriptor of a Q or K tile (e4m3 at d = 64: 64-byte rows)
            auto kdesc = [](uint32_t a) -> uint64_t {
                if constexpr (F8 && D == 64) return sw64_desc(a, 16, 512);
                else return sw128_desc(a, 16, 1024);
            };
            // S_t from the K tile at ring position kpos
            auto issue_S = [&](int t, int kpos) {
                const uint32_t qs = sbase + t * C::kTileBytes;
                const uint32_t ks = slot(kpos % C::kStages);
#pragma unroll
                for (int kk = 0; kk < C::kKSteps; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    if constexpr (F8)
                        mma_ss_f8(tmem + colS[t], kdesc(qs + off), kdesc(ks + off), idS, kk > 0);
                    else
                        mma_ss(tmem + colS[t], sw128_desc(qs + off, 16, 1024), sw128_desc(ks + off, 16, 1024), idS,
                               kk > 0);
                }
                tc_commit(bar(C::kBarS + t));
            };
            // O_t (+)= P_t V, V at ring position vpos; `acc` false for the tile's first P V
            auto issue_PV = [&](int t, int vpos, bool acc) {
                const uint32_t vs = slot(vpos % C::kStages);
                if constexpr (F8) {
                    // A = P_t (shared memory, 128 queries x 128 keys, K-major), B = V (128 keys
                    // x d, MN-major: each 32-key step is 32 rows of d bytes)
                    const uint32_t ps = sbase + C::kOffP + t * 16384;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = (D == 64) ? sw64_desc(vs + kk * 2048, 16384, 512)
                                                         : sw128_desc(vs + kk * 4096, 16384, 1024);
                        mma_ss_f8(tmem + colO[t], sw128_desc(ps + kk * 32, 16, 1024), bdesc, idPV,
                                  (acc || kk > 0) ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tmem + colO[t], tmem + colS[t] + kk * 8, sw128_desc(vs + kk * 2048, 16384, 1024), idPV,
                               (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = true;
            int base = 0;          // ring position of the unit's K_0
            int n_u = 0;           // units started
            int gs[2] = {0, 0};    // S_t products issued (all units): phase counters
            FOR_EACH_UNIT(u, consumer_rank) {
                if (!ok) break;
                const int hi = u.nkv_max();
                int j = u.ufirst<kDiagFirst>();  // the unit's key tiles are j, uafter(j), ... (< hi)
                if (j >= hi) continue;  // no tile pair to compute (tile mask)
                int pos = base;         // ring position of K_j (V_j follows it)
                ok = wait_phase(bar(C::kBarQ), n_u & 1, p.ctl, abort_flag);
                if (ok) ok = wait_phase(bar(C::kBarFull + pos % C::kStages), (pos / C::kStages) & 1, p.ctl, abort_flag);
                if (ok) ok = tag_ok(r_, pos, j);
                if (!ok) break;
                tc_fence_after();
                // The unit's first S_t may overwrite S_t / P_t: PV_t of the previous unit
                // was issued earlier (in-order completion) after its softmax had read S_t.
                for (int t = 0; t < 2; ++t)
                    if (u.live(t, j)) issue_S(t, pos);
                tc_commit(bar(C::kBarEmpty + pos % C::kStages));
                int nxt = u.uafter<kDiagFirst>(j);
                if (nxt >= hi) tc_commit(bar(C::kBarQEmpty));
                bool started[2] = {false, false};
                const int last[2] = {u.ulast<kDiagFirst>(0), u.ulast<kDiagFirst>(1)};
                while (ok) {
                    ok = wait_phase(bar(C::kBarFull + (pos + 1) % C::kStages), ((pos + 1) / C::kStages) & 1, p.ctl,
                                    abort_flag);
                    if (ok) ok = tag_ok(r_, pos + 1, j);
                    if (!ok) break;
                    bool k_next = false;
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (u.live(t, j)) {
                            ok = wait_phase(bar(C::kBarP + t), gs[t] & 1, p.ctl, abort_flag);
                            if (!ok) break;
                            ++gs[t];
                            tc_fence_after();
                            issue_PV(t, pos + 1, started[t]);
                            started[t] = true;
                            if (j == last[t]) tc_commit(bar(C::kBarO + t));
                        }
                        if (nxt < hi && u.live(t, nxt)) {
                            if (!k_next) {
                                ok = wait_phase(bar(C::kBarFull + (pos + 2) % C::kStages), ((pos + 2) / C::kStages) & 1,
                                                p.ctl, abort_flag);
                                if (ok) ok = tag_ok(r_, pos + 2, nxt);
                                if (!ok) break;
                                tc_fence_after();
                                k_next = true;
                            }
                            issue_S(t, pos + 2);
                        }
                    }
                    if (!ok) break;
                    tc_commit(bar(C::kBarEmpty + (pos + 1) % C::kStages));
                    if (k_next) tc_commit(bar(C::kBarEmpty + (pos + 2) % C::kStages));
                    pos += 2;
                    if (nxt >= hi) break;
                    j = nxt;
                    nxt = u.uafter<kDiagFirst>(j);
                    if (nxt >= hi) tc_commit(bar(C::kBarQEmpty));  // the S products just issued were the unit's last
                }
                if (!ok) break;
                base = pos;
                ++n_u;
            }
            if constexpr (kDebugChecks) {
                dbg_cnt[2] = static_cast<uint32_t>(n_u);
                dbg_cnt[3] = static_cast<uint32_t>(base);
                dbg_cnt[4] = static_cast<uint32_t>(gs[0]);
                dbg_cnt[5] = static_cast<uint32_t>(gs[1]);
            }
            // Every MMA issued above must have finished before TMEM / smem go away.
            tc_commit(bar(C::kBarDone));
            drain_phase(bar(C::kBarDone), 0, p.ctl, abort_flag);
        }
    }
    } else {
        setmaxnreg_inc<C::kRegsSoftmax>();
        // ------------------------------------------------------------ softmax warps
        const int t = warp >> 2, q4 = warp & 3;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tmem + lane_off + (t ? C::kColS1 : C::kColS0);
        const uint32_t tO = tmem + lane_off + (t ? C::kColO1 : C::kColO0);
        const float c2 = p.scale_log2;
        bool ok = true;
        int gs = 0;  // S_t phases consumed (all units)
        int go = 0;  // units in which this tile was active
        FOR_EACH_UNIT(u, consumer_rank) {
        if (!ok) break;
        // only what this tile needs is kept from the unit (registers)
        const int len = u.len;
        const int row = u.m0 + 128 * t + q4 * 32 + lane;  // query row within the slice
        const int nkv_t = u.nkv(t);
        const uint8_t *keep = p.g.key_keep ? p.g.key_keep + p.g.keep_base(u.b, u.start) : nullptr;
        float m_used = -INFINITY, l = 0.f;
        const TileSet ts = t ? u.ts1 : u.ts0;  // the key tiles this tile attends
        bool first_step = true;
        // (Q1 with its diagonal tile first: see FwdUnit::ufirst)
        const bool df = kDiagFirst && t == 1 && u.diag_first;
        for (int j = df ? ts.hi - 1 : ts.next(0); j < ts.hi;
             j = df ? (j == ts.hi - 1 ? (ts.hi > 1 ? 0 : ts.hi) : (j + 1 < ts.hi - 1 ? j + 1 : ts.hi)) : ts.next(j + 1),
             ++gs) {
            const int kbase = j * 128;
            ok = wait_phase(bar(C::kBarS + t), gs & 1, p.ctl, abort_flag);
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, sr[q]);
            tmem_wait_ld();
            float s[128];
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);

            // ---- masking: keys outside the sequence, above the diagonal, or padded
            int limit = len - kbase;
            if (p.causal) limit = min(limit, row - kbase + 1);
            if (limit < 128) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= limit) s[c] = -INFINITY;
            }
            if (keep != nullptr) {
                const int kl = len - kbase;  // keys of this tile inside the sequence
                uint32_t kmask[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int c = q * 32 + lane;
                    const bool kept = (c < kl) && keep[kbase + c] != 0;
                    kmask[q] = __ballot_sync(0xffffffffu, kept);
                }
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (!((kmask[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
            }

            // ---- running max with lazy correction
            // four independent 3-input max chains (short dependency chains: one warp per
            // scheduler runs this, so latency, not issue rate, is what matters)
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 128; c += 8) {
#pragma unroll
                for (int u = 0; u < 4; ++u) mq[u] = fmax3(mq[u], s[c + 2 * u], s[c + 2 * u + 1]);
            }
            const float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
            const float m_cand = mx * c2;
            const bool need = m_cand > m_used + kRescaleThreshold;
            const bool warp_rescale = __any_sync(0xffffffffu, need);
            float alpha = 1.f;
            if (need) {
                alpha = ex2_approx(m_used - m_cand);  // m_used == -inf gives 0
                m_used = m_cand;
                l *= alpha;
            }
            const float m_use = (m_used == -INFINITY) ? 0.f : m_used;

            // ---- probabilities (bf16) into TMEM over S, and the row sum.  Column pairs
            // go through the packed f32x2 pipe: one instruction scales and shifts both
            // scores, one adds both probabilities to a pair of running sums.
            const uint64_t c2x2 = f2_pack(c2, c2), negm2 = f2_pack(-m_use, -m_use);
            uint64_t ps2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const uint64_t x2 = f2_fma(f2_pack(s[half * 64 + 2 * c], s[half * 64 + 2 * c + 1]), c2x2, negm2);
                    float p0, p1;
                    if ((C::kPolyPairs >> (c & 7)) & 1u) {
                        // Where the products take half the time of the exponentials (e4m3
                        // operands at d = 128, bf16 at d = 64) the MUFU unit sets the pace, so
                        // some column pairs go to the FMA pipe
                        ex2_poly_x2(x2, p0, p1);
                    } else {
                        float x0, x1;
                        f2_unpack(x2, x0, x1);
                        p0 = ex2_approx(x0);
                        p1 = ex2_approx(x1);
                    }
                    ps2[c & 1] = f2_add(ps2[c & 1], f2_pack(p0, p1));
                    if constexpr (F8) {
                        const uint32_t h2 = pack_e4m3x2(p0, p1);
                        pk[c >> 1] = (c & 1) ? (pk[c >> 1] | (h2 << 16)) : h2;
                    } else {
                        pk[c] = pack_bf16x2(p0, p1);
                    }
                }
                if constexpr (F8) {
                    // this row's 64 keys as 4 chunks of 16 bytes, at the 128-byte-swizzle
                    // positions of a K-major tile (chunk c of row r at r*128 + ((c ^ r%8) * 16))
                    const int r = q4 * 32 + lane;
                    const uint32_t prow = sbase + C::kOffP + t * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        st_shared_v4(prow + ((((half * 4 + cc) ^ (r & 7)) & 7) << 4), pk[4 * cc], pk[4 * cc + 1],
                                     pk[4 * cc + 2], pk[4 * cc + 3]);
                } else {
                    tmem_st32(tS + half * 32, pk);
                }
            }
            {
                float a0, a1, b0, b1;
                f2_unpack(ps2[0], a0, a1);
                f2_unpack(ps2[1], b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            // Lazy correction of O_t, after the scores are dead (fewer live registers)
            // but before P_t is published: PV_t(j) is issued only after the arrive.
            if (warp_rescale && !first_step) {
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t orr[32];
                    tmem_ld32(tO + q * 32, orr);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
                    tmem_st32(tO + q * 32, orr);
                }
            }
            tmem_wait_st();
            if constexpr (F8) fence_proxy_async_smem();  // P_t is read by the tensor core (async proxy)
            tc_fence_before();
            mbar_arrive(bar(C::kBarP + t));
            first_step = false;
        }

        // ---- epilogue: O / l in bf16, lse in natural log.  The next unit's PV_t(0),
        // which overwrites O_t, is issued only after this thread's next P_t arrive.
        if (ok && nkv_t > 0 && first_step) {
            // The tile mask leaves this tile no key tile: O = 0 and lse = -inf, like any
            // row that sees no key; nothing was computed for it.
            FwdUnit e;
            fwd_unit<SP, NT, DYN, false>(p, kDyn ? r_ : static_rank(k_), e);  // (static: recomputed, not kept live)
            if (row < len) {
                const long long r = static_cast<long long>(row);
                uint4 *dst = reinterpret_cast<uint4 *>(p.o + p.g.base(e.b, e.h, e.start, D) + r * p.g.row_stride(D));
#pragma unroll 1
                for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                p.lse[p.g.base(e.b, e.h, e.start, 1) + r * p.g.row_stride(1)] = -INFINITY;
            }
            continue;
        }
        if (ok && nkv_t > 0) ok = wait_phase(bar(C::kBarO + t), go & 1, p.ctl, abort_flag);
        if (ok && nkv_t > 0) {
            ++go;
            tc_fence_after();
            const bool valid = row < len;
            const float inv = (l > 0.f) ? p.o_scale / l : 0.f;
            const float lse_v = (l > 0.f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
            FwdUnit e;  // the unit again, from the loop counter (fewer registers live in the key loop)
            fwd_unit<SP, NT, DYN, false>(p, kDyn ? r_ : static_rank(k_), e);  // (static: recomputed, not kept live)
            __nv_bfloat16 *orow = p.o + p.g.base(e.b, e.h, e.start, D) + static_cast<long long>(row) * p.g.row_stride(D);
            // A warp's full 32-row block goes out by TMA store from its stage (laid out
            // as the 64-byte swizzle of a 32 x 32 box), so the warp moves on to the next
            // unit without waiting for the global writes; a block reaching past the
            // sequence's end (which a packed layout could not clip) is stored row by row.
            const int row_w0 = row - lane;
            // (one tile per CTA at d = 64: direct stores, whose latency the other CTA of the SM
            // hides; measured 4 % faster there, neutral at d = 128)
            const bool by_tma = (NT == 2 || D == 128) && len - row_w0 >= 32;
            const uint32_t stage = sbase + C::kOffStage + warp * 2048;
#pragma unroll 1  // (unrolled, the 128-wide key loop above runs out of registers)
            for (int q = 0; q < D / 32; ++q) {
                uint32_t orr[32];
                tmem_ld32(tO + q * 32, orr);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    pk[c] = pack_bf16x2(__uint_as_float(orr[2 * c]) * inv, __uint_as_float(orr[2 * c + 1]) * inv);
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
                        tma_store_3d(&tm_o_st, stage, q * 32, p.g.tma_row0(e.start) + row_w0, p.g.tma_slab(e.b, e.h));
                        bulk_commit();
                    }
                } else if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + q * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
            }
            if (valid) p.lse[p.g.base(e.b, e.h, e.start, 1) + static_cast<long long>(row) * p.g.row_stride(1)] = lse_v;
        }
        }
        if (lane == 0) bulk_wait0();  // this warp's output stores are complete
        if constexpr (kDebugChecks)
            if (q4 == 0 && lane == 0) dbg_cnt[6 + t] = static_cast<uint32_t>(gs);
    }
#undef FOR_EACH_UNIT

    __syncwarp();  // reconverge the single-lane roles before the CTA barrier
    tc_fence_before();
    __syncthreads();
    if (warp == C::kProducerWarp && lane == 0 && *abort_flag) {
        // After an abort, every copy the producer started must land before the CTA
        // exits (the flag is final here: every role has finished).
        for (int s = 0; s < C::kStages; ++s) {
            int last = n_issued - 1 - ((n_issued - 1 - s) % C::kStages + C::kStages) % C::kStages;
            if (last == p.ctl.inject_skip_load) last -= C::kStages;
            if (last >= 0) drain_phase(bar(C::kBarFull + s), (last / C::kStages) & 1, p.ctl, abort_flag);
        }
        if (n_qload > 0) drain_phase(bar(C::kBarQ), (n_qload - 1) & 1, p.ctl, abort_flag);
    }
    if (warp == C::kIssuerWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if constexpr (kDebugChecks) {
        // without an abort, every role walked the same units, fills and S phases
        if (threadIdx.x == 0 && !*abort_flag) {
            bool agree = dbg_cnt[0] == dbg_cnt[2] && dbg_cnt[1] == dbg_cnt[3] && dbg_cnt[4] == dbg_cnt[6];
            if (NT == 2) agree = agree && dbg_cnt[5] == dbg_cnt[7];
            if (!agree) atomicCAS(p.ctl.status, 0, kStatusDebugCheck);
        }
    }
    if constexpr (kDyn) {
        // the last CTA to finish returns the counters to zero for the slot's next launch
        if (threadIdx.x == 0) {
            __threadfence();
            if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
                atomicExch(p.sched, 0u);
                atomicExch(p.sched + 1, 0u);
            }
        }
    }
}

template <int D, bool SP, bool F8 = false, int NT = 2, bool DYN = false>
static cudaError_t launch_fwd_d(const FwdLaunch &a, cudaStream_t stream) {
    using C = FwdCfg<D, F8, NT>;
    FwdParams p{};
    p.g = a.g;
    p.ctl = a.ctl;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.lse = a.lse;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.o_scale = 1.f;
    if constexpr (F8) {
        p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * a.q_scale * a.k_scale * 1.4426950408889634);
        p.o_scale = a.v_scale;
    }
    p.causal = a.causal;
    p.n_units = (a.g.N + 128 * NT - 1) / (128 * NT);
    p.sched = nullptr;
    // K and V of a slice; banded only beyond about twice the L2 cache
    p.band = l2_band(a.g.B * a.g.H, 2.0 * a.g.N * a.g.d * C::kEsz, 256.0 * 1024 * 1024);
    if (forced_band() > 0) p.band = min(forced_band(), a.g.B * a.g.H);  // (test hook; DYN kernels only)
    if constexpr (DYN) {
        p.sched = next_sched_slot();
        if (p.sched == nullptr) return cudaErrorInvalidSymbol;
    }
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_sm100_kernel<D, SP, F8, NT, DYN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // The in-kernel register reallocation assumes the launch register count it was
    // sized for; with fewer, an increase could never be satisfied, so refuse.
    static const cudaError_t regs_ok = [] {
        cudaFuncAttributes fa{};
        const cudaError_t r = cudaFuncGetAttributes(&fa, attn_fwd_sm100_kernel<D, SP, F8, NT, DYN>);
        if (r != cudaSuccess) return r;
        return fa.numRegs == C::kLaunchRegs ? cudaSuccess : cudaErrorInvalidKernelImage;
    }();
    if (regs_ok != cudaSuccess) return regs_ok;
    const long long units = static_cast<long long>(a.g.B) * a.g.H * p.n_units;
    const long long slots = static_cast<long long>(a.num_sms) * C::kCtasPerSm;
    const dim3 grid(static_cast<unsigned>(units < slots ? units : slots));
    attn_fwd_sm100_kernel<D, SP, F8, NT, DYN><<<grid, C::kThreads, C::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_o_st,
                                                                                    p);
    return cudaGetLastError();
}

cudaError_t launch_fwd_fp8(const FwdLaunch &a, cudaStream_t stream) {
    const bool dyn = a.g.varlen != 0;  // packed sequences: uneven units, claimed at run time
    // a tile mask: one query tile per CTA, two CTAs per SM, units claimed at run time
    // (as the bf16 kernel)
    const bool sp = a.g.block_mask != nullptr;
    if (a.g.d == 128) {
        if (sp) return launch_fwd_d<128, true, true, 1, true>(a, stream);
        return dyn ? launch_fwd_d<128, false, true, 2, true>(a, stream) : launch_fwd_d<128, false, true>(a, stream);
    }
    if (a.g.d == 64) {
        if (sp) return launch_fwd_d<64, true, true, 1, true>(a, stream);
        return dyn ? launch_fwd_d<64, false, true, 2, true>(a, stream) : launch_fwd_d<64, false, true>(a, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fwd(const FwdLaunch &a, cudaStream_t stream) {
    const bool sp = a.g.block_mask != nullptr;
    // a tile mask: one query tile per CTA, two CTAs per SM
    const bool dyn = a.g.varlen != 0;  // packed sequences: uneven units, claimed at run time
    if (a.g.d == 128) {
        if (sp) return launch_fwd_d<128, true, false, 1, true>(a, stream);
        return dyn ? launch_fwd_d<128, false, false, 2, true>(a, stream) : launch_fwd_d<128, false>(a, stream);
    }
    if (sp) return launch_fwd_d<64, true, false, 1, true>(a, stream);
    return dyn ? launch_fwd_d<64, false, false, 2, true>(a, stream) : launch_fwd_d<64, false>(a, stream);
}

}  // namespace attn
