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
// Three launches on one stream:
//   1. attn_bwd_pre_kernel   D_i, lse2_i = lse_i log2(e) (+inf for rows that saw no
//                            key, so their recomputed P is exactly 0), and a zeroed
//                            fp32 dQ accumulator.  HBM-bound, vectorised.
//   2. attn_bwd_main_kernel  one CTA per 128-key tile of one (sequence, head); it
//                            keeps K_j, V_j in shared memory and sweeps the 64-row
//                            query tiles i (only i >= the diagonal when causal):
//        S^T  = K_j Q_i^T      (tcgen05, M=128 keys, N=64 queries)  -> TMEM
//        dP^T = V_j dO_i^T     (tcgen05, M=128, N=64)               -> TMEM
//        P^T  = 2^(S^T scale log2e - lse2), dS^T = P^T o (dP^T - D) by 8 warps,
//               written as bf16 into 128-byte-swizzled shared-memory tiles
//        (Q_i, dO_i and their row terms sit in a 3-stage ring so the next tiles'
//         loads are in flight a full iteration before they are needed)
//        dV  += P^T  dO_i      (M=128, N=d, K=64)                   -> TMEM
//        dK  += dS^T Q_i       (M=128, N=d, K=64)                   -> TMEM
//        dQ_i = dS K_j         (M=64,  N=d, K=128)                  -> TMEM, then
//               staged in shared memory by 4 warps and added into the fp32
//               accumulator with bulk tensor reduce-adds (TMA)
//      and finally writes dV and scale*dK in bf16.
//   3. attn_bwd_dq_kernel    dQ = bf16(scale * accumulator).  HBM-bound.
//
// Tensor memory of the main kernel (columns): S^T [0,64), dP^T [64,128),
// dQ [128,128+d), dV [128+d,128+2d), dK [128+2d,128+3d): no region is shared, so
// the next tile's S^T / dP^T products are issued as soon as the softmax warps have
// copied the current ones into registers, and overlap its softmax work.
//
// Warp roles (448 threads): warps 0-7 probabilities/dS (warp w: key rows
// 32*(w%4).., query columns 32*(w/4)..), warps 8-11 dQ drain (thread 256 issues
// the bulk reductions) and the dK/dV
// epilogue, warp 12 loader (TMA for K, V, Q, dO; plain loads for lse2/D),
// warp 13 TMEM allocator and MMA issuer.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "attn_common.cuh"
#include "attn_launch.h"

namespace attn {

constexpr float kLog2e = 1.4426950408889634f;

// ============================================================================ preprocess
// One row of d elements per (d/8) threads.  Rows are in the lse layout order,
// which is also the row order of the flat [rows, d] view of O and dO.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(const __nv_bfloat16 *__restrict__ o,
                                                          const __nv_bfloat16 *__restrict__ dout,
                                                          const float *__restrict__ lse, float *__restrict__ dvec,
                                                          float *__restrict__ lse2, float *__restrict__ dq_acc,
                                                          long long rows, const int32_t *cu_seqlens, int nseq,
                                                          int H) {
    constexpr int TPR = D / 8;  // threads per row
    long long limit = rows;
    if (cu_seqlens) limit = min(rows, static_cast<long long>(cu_seqlens[nseq]) * H);
    const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long row = gt / TPR;
    const int part = static_cast<int>(gt % TPR);
    const bool active = row < limit;
    float acc = 0.f;
    if (active) {
        const uint4 a = *reinterpret_cast<const uint4 *>(o + row * D + part * 8);
        const uint4 g = *reinterpret_cast<const uint4 *>(dout + row * D + part * 8);
        const __nv_bfloat162 *a2 = reinterpret_cast<const __nv_bfloat162 *>(&a);
        const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&g);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(a2[e]);
            const float2 y = __bfloat1622float2(g2[e]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
        float4 *z = reinterpret_cast<float4 *>(dq_acc + row * D + part * 8);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (active && part == 0) {
        dvec[row] = acc;
        const float L = lse[row];
        lse2[row] = (L == -INFINITY) ? INFINITY : L * kLog2e;
    }
}

// ============================================================================ dQ finish
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float *__restrict__ dq_acc,
                                                         __nv_bfloat16 *__restrict__ dq, long long rows, float scale,
                                                         const int32_t *cu_seqlens, int nseq, int H) {
    long long limit = rows;
    if (cu_seqlens) limit = min(rows, static_cast<long long>(cu_seqlens[nseq]) * H);
    const long long n8 = limit * D / 8;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float4 a = reinterpret_cast<const float4 *>(dq_acc)[2 * i];
        const float4 b = reinterpret_cast<const float4 *>(dq_acc)[2 * i + 1];
        uint4 r;
        r.x = pack_bf16x2(a.x * scale, a.y * scale);
        r.y = pack_bf16x2(a.z * scale, a.w * scale);
        r.z = pack_bf16x2(b.x * scale, b.y * scale);
        r.w = pack_bf16x2(b.z * scale, b.w * scale);
        reinterpret_cast<uint4 *>(dq)[i] = r;
    }
}

// ============================================================================ main kernel
template <int D>
struct BwdCfg {
    static constexpr int kKVBytes = 128 * D * 2;  // K_j or V_j (128 rows)
    static constexpr int kQBytes = 64 * D * 2;    // Q_i or dO_i (64 rows)
    static constexpr int kKVBox = 128 * 128;      // one 64-column box of a 128-row tile
    static constexpr int kQBox = 64 * 128;        // one 64-column box of a 64-row tile
    static constexpr int kBoxes = D / 64;
    static constexpr int kPSBytes = 128 * 128;    // P^T or dS^T: 128 keys x 64 queries bf16
    static constexpr int kStages = 3;             // Q/dO/vector stages (load latency stays hidden)
    static constexpr int kThreads = 448;
    static constexpr int kTmemCols = 512;
    static constexpr int kColS = 0, kColDP = 64, kColDQ = 128, kColDV = 128 + D, kColDK = 128 + 2 * D;
    // shared-memory offsets (from the 1024-aligned base)
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kKVBytes;
    static constexpr int kOffQ = 2 * kKVBytes;                         // + st * kQBytes
    static constexpr int kOffDO = kOffQ + kStages * kQBytes;           // + st * kQBytes
    static constexpr int kOffP = kOffDO + kStages * kQBytes;           // P^T tile (single buffer)
    static constexpr int kOffDS = kOffP + kPSBytes;                    // dS^T tile (single buffer)
    static constexpr int kOffDQ = kOffDS + kPSBytes;                   // fp32 dQ stage: d/32 boxes of 64x32
    static constexpr int kDQBox = 64 * 128;
    static constexpr int kOffVec = kOffDQ + (D / 32) * kDQBox;         // + st * 512: lse2[64], D[64]
    static constexpr int kOffBar = kOffVec + kStages * 512;
    // every swizzled tile must start on a 1024-byte boundary
    static_assert(kOffQ % 1024 == 0 && kOffDO % 1024 == 0 && kOffP % 1024 == 0 && kOffDS % 1024 == 0 &&
                      kOffDQ % 1024 == 0 && kQBytes % 1024 == 0,
                  "swizzled shared-memory tiles must be 1024-byte aligned");
    // barriers
    static constexpr int kBarKV = 0;
    static constexpr int kBarQFull = 1;                 // + st
    static constexpr int kBarQEmpty = 1 + kStages;      // + st
    static constexpr int kBarSdpFull = 1 + 2 * kStages;
    static constexpr int kBarSdpFree = 2 + 2 * kStages;
    static constexpr int kBarPsFull = 3 + 2 * kStages;  // P^T and dS^T written (256 threads)
    static constexpr int kBarPsEmpty = 4 + 2 * kStages; // dV, dK, dQ finished reading them
    static constexpr int kBarDqFull = 5 + 2 * kStages;
    static constexpr int kBarDqEmpty = 6 + 2 * kStages;
    static constexpr int kBarKdv = 7 + 2 * kStages;
    static constexpr int kBarDone = 8 + 2 * kStages;
    static constexpr int kBarStageFull = 9 + 2 * kStages;   // dQ stage written (128 drain threads)
    static constexpr int kBarStageFree = 10 + 2 * kStages;  // dQ stage read by the bulk reduce (leader)
    static constexpr int kNumBars = 11 + 2 * kStages;
    static constexpr int kSmemBytes = 1024 + kOffBar + kNumBars * 8 + 16;
    static_assert(kSmemBytes <= 232448, "exceeds the 227 KB per-CTA shared-memory limit");
};

struct BwdParams {
    Geom g;
    SyncCtl ctl;
    __nv_bfloat16 *dk, *dv;
    float *dq_acc;
    const float *dvec, *lse2;
    float scale;
    float scale_log2;
    int causal;
    int n_kv;  // 128-key tiles per slice (grid z)
};

template <int D>
__global__ void __launch_bounds__(448, 1)
attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dqacc, const __grid_constant__ BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    uint8_t *sptr = smem_raw + (sbase - raw_u32);
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sptr + C::kOffBar + C::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, b = blockIdx.y, j = blockIdx.z;  // small j (most query tiles) first
    int start, len;
    p.g.slice(b, start, len);
    const int kv0 = j * 128;
    if (kv0 >= len) return;  // uniform, before any barrier or allocation
    const int nq_all = (len + 63) / 64;
    const int i0 = p.causal ? (kv0 / 64) : 0;
    const int nq = nq_all - i0;  // >= 1

    if (warp == 13) {
        tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i == C::kBarSdpFree || i == C::kBarPsFull) cnt = 256;
            if (i == C::kBarDqEmpty || i == C::kBarStageFull) cnt = 128;
            mbar_init(bar(i), cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const long long lrow0 = p.g.base(b, h, start, 1);
    const long long lrs = p.g.row_stride(1);
    int n_issued = 0;  // loader: query-tile loads 0 .. n_issued-1 were started

    if (warp == 12) {
        // ------------------------------------------------------------ loader
        const int row0 = p.g.tma_row0(start), slab = p.g.tma_slab(b, h);
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            mbar_arrive_expect_tx(bar(C::kBarKV), 2 * C::kKVBytes);
#pragma unroll
            for (int x = 0; x < C::kBoxes; ++x) {
                tma_load_3d(sbase + C::kOffK + x * C::kKVBox, &tm_k, bar(C::kBarKV), x * 64, row0 + kv0, slab);
                tma_load_3d(sbase + C::kOffV + x * C::kKVBox, &tm_v, bar(C::kBarKV), x * 64, row0 + kv0, slab);
            }
        }
        for (int it = 0; it < nq; ++it) {
            const int st = it % C::kStages;
            const bool ok = __all_sync(
                0xffffffffu, wait_phase(bar(C::kBarQEmpty + st), ((it / C::kStages) & 1) ^ 1, p.ctl, abort_flag));
            if (!ok) break;
            const int q0 = (i0 + it) * 64;
            float *vec = reinterpret_cast<float *>(sptr + C::kOffVec + st * 512);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int q = q0 + u * 32 + lane;
                float l2 = INFINITY, dd = 0.f;  // rows past the sequence: P = 0
                if (q < len) {
                    l2 = p.lse2[lrow0 + q * lrs];
                    dd = p.dvec[lrow0 + q * lrs];
                }
                vec[u * 32 + lane] = l2;
                vec[64 + u * 32 + lane] = dd;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(C::kBarQFull + st), 2 * C::kQBytes);
#pragma unroll
                for (int x = 0; x < C::kBoxes; ++x) {
                    tma_load_3d(sbase + C::kOffQ + st * C::kQBytes + x * C::kQBox, &tm_q, bar(C::kBarQFull + st),
                                x * 64, row0 + q0, slab);
                    tma_load_3d(sbase + C::kOffDO + st * C::kQBytes + x * C::kQBox, &tm_do, bar(C::kBarQFull + st),
                                x * 64, row0 + q0, slab);
                }
            }
            n_issued = it + 1;
        }
    } else if (warp == 13) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idSP = idesc_bf16_f32(128, 64, 0, 0);  // S^T, dP^T
            constexpr uint32_t idKV = idesc_bf16_f32(128, D, 0, 1);   // dV, dK
            constexpr uint32_t idQ = idesc_bf16_f32(64, D, 1, 1);     // dQ
            auto issue_sdp = [&](int it) {
                const int st = it % C::kStages;
                const uint32_t qs = sbase + C::kOffQ + st * C::kQBytes;
                const uint32_t ds = sbase + C::kOffDO + st * C::kQBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t okv = (kk >> 2) * C::kKVBox + (kk & 3) * 32;
                    const uint32_t oq = (kk >> 2) * C::kQBox + (kk & 3) * 32;
                    mma_ss(tmem + C::kColS, sw128_desc(sbase + C::kOffK + okv, 16, 1024), sw128_desc(qs + oq, 16, 1024),
                           idSP, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t okv = (kk >> 2) * C::kKVBox + (kk & 3) * 32;
                    const uint32_t oq = (kk >> 2) * C::kQBox + (kk & 3) * 32;
                    mma_ss(tmem + C::kColDP, sw128_desc(sbase + C::kOffV + okv, 16, 1024),
                           sw128_desc(ds + oq, 16, 1024), idSP, kk > 0);
                }
                tc_commit(bar(C::kBarSdpFull));
            };
            bool ok = wait_phase(bar(C::kBarKV), 0, p.ctl, abort_flag);
            if (ok) ok = wait_phase(bar(C::kBarQFull + 0), 0, p.ctl, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_sdp(0);
            }
            for (int it = 0; ok && it < nq; ++it) {
                const int st = it % C::kStages;
                if (it + 1 < nq) {
                    const int nx = it + 1;
                    ok = wait_phase(bar(C::kBarQFull + nx % C::kStages), (nx / C::kStages) & 1, p.ctl, abort_flag);
                    if (ok) ok = wait_phase(bar(C::kBarSdpFree), it & 1, p.ctl, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_sdp(it + 1);
                }
                ok = wait_phase(bar(C::kBarPsFull), it & 1, p.ctl, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t ps = sbase + C::kOffP;
                const uint32_t dss = sbase + C::kOffDS;
                const uint32_t qs = sbase + C::kOffQ + st * C::kQBytes;
                const uint32_t dos = sbase + C::kOffDO + st * C::kQBytes;
                // dV += P^T dO_i ; dK += dS^T Q_i   (K = 64 queries, 4 steps)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem + C::kColDV, sw128_desc(ps + kk * 32, 16, 1024),
                           sw128_desc(dos + kk * 2048, C::kQBox, 1024), idKV, (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem + C::kColDK, sw128_desc(dss + kk * 32, 16, 1024),
                           sw128_desc(qs + kk * 2048, C::kQBox, 1024), idKV, (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(bar(C::kBarQEmpty + st));
                // dQ_i = dS K_j   (M = 64 queries, K = 128 keys, 8 steps); the drain
                // warps must have emptied the previous dQ tile first.
                ok = wait_phase(bar(C::kBarDqEmpty), (it & 1) ^ 1, p.ctl, abort_flag);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmem + C::kColDQ, sw128_desc(dss + kk * 2048, 8192, 1024),
                           sw128_desc(sbase + C::kOffK + kk * 2048, C::kKVBox, 1024), idQ, kk > 0);
                tc_commit(bar(C::kBarDqFull));
                tc_commit(bar(C::kBarPsEmpty));
            }
            if (ok) tc_commit(bar(C::kBarKdv));
            tc_commit(bar(C::kBarDone));
            drain_phase(bar(C::kBarDone), 0, p.ctl, abort_flag);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ P^T and dS^T
        const int q4 = warp & 3, hf = warp >> 2;
        const int kr = q4 * 32 + lane;  // key row within the tile
        const int key = kv0 + kr;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        bool kvalid = key < len;
        if (kvalid && p.g.key_keep) kvalid = p.g.key_keep[p.g.keep_base(b, start) + key] != 0;
        const float c2 = p.scale_log2;
        for (int it = 0; it < nq; ++it) {
            const int st = it % C::kStages;
            bool ok = wait_phase(bar(C::kBarSdpFull), it & 1, p.ctl, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[32], dpr[32];
            tmem_ld32(tmem + lane_off + C::kColS + hf * 32, sr);
            tmem_ld32(tmem + lane_off + C::kColDP + hf * 32, dpr);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(C::kBarSdpFree));
            ok = __all_sync(0xffffffffu,
                            wait_phase(bar(C::kBarQFull + st), (it / C::kStages) & 1, p.ctl, abort_flag));
            if (!ok) break;
            const float *vec = reinterpret_cast<const float *>(sptr + C::kOffVec + st * 512);
            const int qb = (i0 + it) * 64 + hf * 32;  // first query column of this warp
            int lim = p.causal ? key - qb : 0;         // columns c < lim have query < key
            if (!kvalid) lim = 32;
            uint32_t pp[16], dsp[16];
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                float pr[2], dsv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cc = c + e;
                    const float l2 = vec[hf * 32 + cc];
                    const float dd = vec[64 + hf * 32 + cc];
                    float pv = ex2_approx(fmaf(__uint_as_float(sr[cc]), c2, -l2));
                    if (cc < lim) pv = 0.f;
                    pr[e] = pv;
                    dsv[e] = pv * (__uint_as_float(dpr[cc]) - dd);
                }
                pp[c >> 1] = pack_bf16x2(pr[0], pr[1]);
                dsp[c >> 1] = pack_bf16x2(dsv[0], dsv[1]);
            }
            ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarPsEmpty), (it & 1) ^ 1, p.ctl, abort_flag));
            if (!ok) break;
            // 128-byte swizzled K-major rows: 16-byte chunk c of row r sits at chunk c ^ (r & 7)
            const uint32_t prow = sbase + C::kOffP + kr * 128;
            const uint32_t drow = sbase + C::kOffDS + kr * 128;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t chunk = static_cast<uint32_t>((hf * 4 + u) ^ (kr & 7)) << 4;
                st_shared_v4(prow + chunk, pp[4 * u], pp[4 * u + 1], pp[4 * u + 2], pp[4 * u + 3]);
                st_shared_v4(drow + chunk, dsp[4 * u], dsp[4 * u + 1], dsp[4 * u + 2], dsp[4 * u + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(C::kBarPsFull));
        }
    } else {
        // ------------------------------------------------------------ dQ drain + dK/dV epilogue
        // Each dQ_i tile (fp32, M = 64) goes TMEM -> registers -> a 128-byte swizzled
        // shared-memory stage -> one bulk tensor reduce-add per 32-column box into the
        // fp32 accumulator (the L2 does the additions line by line).  Query rows past
        // the sequence hold exact zeros (their P is 0), so adding them is harmless.
        const int q4 = warp & 3;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const bool leader = threadIdx.x == 256;
        const int row0 = p.g.tma_row0(start), slab = p.g.tma_slab(b, h);
        const uint32_t stage = sbase + C::kOffDQ;
        const int r = q4 * 16 + lane;  // M = 64 accumulator: row r sits in TMEM lane (r % 16) + 32 * (r / 16)
        bool ok = true;
        for (int it = 0; it < nq; ++it) {
            ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarDqFull), it & 1, p.ctl, abort_flag));
            if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarStageFree), (it & 1) ^ 1, p.ctl, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int x = 0; x < D / 32; ++x) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + C::kColDQ + x * 32, v);
                tmem_wait_ld();
                if (x == D / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarDqEmpty));
                }
                if (lane < 16) {
                    const uint32_t rowa = stage + x * C::kDQBox + r * 128;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        st_shared_v4(rowa + ((static_cast<uint32_t>(k ^ (r & 7))) << 4), v[4 * k], v[4 * k + 1],
                                     v[4 * k + 2], v[4 * k + 3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(C::kBarStageFull));
            if (leader) {
                ok = wait_phase(bar(C::kBarStageFull), it & 1, p.ctl, abort_flag);
                if (ok) {
                    const int q0 = (i0 + it) * 64;
#pragma unroll
                    for (int x = 0; x < D / 32; ++x) tma_reduce_add_3d(&tm_dqacc, stage + x * C::kDQBox, x * 32, row0 + q0, slab);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(bar(C::kBarStageFree));
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
        }
        if (leader) bulk_wait0();  // the accumulator updates are complete before the CTA exits
        if (ok) ok = __all_sync(0xffffffffu, wait_phase(bar(C::kBarKdv), 0, p.ctl, abort_flag));
        if (ok) {
            tc_fence_after();
            const int key = kv0 + q4 * 32 + lane;
            const bool valid = key < len;
            const long long off = p.g.base(b, h, start, D) + static_cast<long long>(key) * p.g.row_stride(D);
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                __nv_bfloat16 *out = (which == 0 ? p.dv : p.dk) + off;
                const float mul = which == 0 ? 1.f : p.scale;
                const uint32_t col = which == 0 ? C::kColDV : C::kColDK;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + col + c0, r);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        pk[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * mul, __uint_as_float(r[2 * c + 1]) * mul);
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(out + c0);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 12 && lane == 0 && *abort_flag) {
        // After an abort, every copy the loader started must land before the CTA exits.
        drain_phase(bar(C::kBarKV), 0, p.ctl, abort_flag);
        for (int it = max(0, n_issued - C::kStages); it < n_issued; ++it)
            drain_phase(bar(C::kBarQFull + it % C::kStages), (it / C::kStages) & 1, p.ctl, abort_flag);
    }
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D>
static cudaError_t launch_bwd_d(const BwdLaunch &a, cudaStream_t stream) {
    using C = BwdCfg<D>;
    const int nseq = a.g.B;
    const int *cu = a.g.varlen ? a.g.cu_seqlens : nullptr;
    if (a.phases & 1) {
        const long long threads = a.rows_total * (D / 8);
        const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
        attn_bwd_pre_kernel<D><<<blocks, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(a.o), static_cast<const __nv_bfloat16 *>(a.dout), a.lse, a.dvec,
            a.lse2, a.dq_acc, a.rows_total, cu, nseq, a.g.H);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.phases & 2) {
        BwdParams p{};
        p.g = a.g;
        p.ctl = a.ctl;
        p.dk = static_cast<__nv_bfloat16 *>(a.dk);
        p.dv = static_cast<__nv_bfloat16 *>(a.dv);
        p.dq_acc = a.dq_acc;
        p.dvec = a.dvec;
        p.lse2 = a.lse2;
        p.scale = a.scale;
        p.scale_log2 = a.scale * kLog2e;
        p.causal = a.causal;
        p.n_kv = (a.g.N + 127) / 128;
        cudaError_t e = cudaFuncSetAttribute(attn_bwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        dim3 grid(a.g.H, a.g.B, p.n_kv);
        attn_bwd_main_kernel<D><<<grid, C::kThreads, C::kSmemBytes, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_do,
                                                                             a.tm_dqacc, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.phases & 4) {
        const long long n8 = a.rows_total * D / 8;
        long long blocks = (n8 + 255) / 256;
        if (blocks > 148LL * 64) blocks = 148LL * 64;
        if (blocks < 1) blocks = 1;
        attn_bwd_dq_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
            a.dq_acc, static_cast<__nv_bfloat16 *>(a.dq), a.rows_total, a.scale, cu, nseq, a.g.H);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

cudaError_t launch_bwd(const BwdLaunch &a, cudaStream_t stream) {
    if (a.g.d == 128) return launch_bwd_d<128>(a, stream);
    return launch_bwd_d<64>(a, stream);
}

}  // namespace attn
