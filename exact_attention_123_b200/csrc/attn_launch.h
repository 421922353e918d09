// attn_launch.h -- host-side launch descriptors passed from the C ABI layer to the
// kernel launchers.  Internal to the library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "attn_common.cuh"

namespace attn {

struct FwdLaunch {
    CUtensorMap tm_q, tm_k, tm_v;  // 3-D bf16 maps, box {64, 128, 1}, 128-byte swizzle
    CUtensorMap tm_o_st;           // O stores: box {32, 32, 1}, 64-byte swizzle
    Geom g;
    SyncCtl ctl;
    void *o;
    float *lse;
    float scale;
    int causal;
    int num_sms;  // persistent grid size
    float q_scale, k_scale, v_scale;  // e4m3 forward only: dequantisation factors
};

struct BwdLaunch {
    CUtensorMap tm_q, tm_k, tm_v, tm_do;  // same map shape as the forward (128-row boxes)
    CUtensorMap tm_dk_st, tm_dv_st;       // dK, dV stores: 32 x 32 boxes, 64-byte swizzle
    CUtensorMap tm_dqacc;                 // fp32 dQ accumulator reduce-adds: 32 x 32 boxes, 128-byte swizzle
    Geom g;
    SyncCtl ctl;
    const void *o, *dout;
    const float *lse;
    void *dq, *dk, *dv;
    float *dvec;       // fp32 D_i = rowsum(dO o O), lse layout (workspace)
    float *lse2;       // fp32 lse * log2(e), +inf for empty rows, lse layout (workspace)
    float *dqacc;      // fp32 dQ accumulator, q's layout (workspace; single-pass backward only)
    long long rows_total;  // token rows (packed) or B*H*N (dense) of the lse layout
    float scale;
    int causal;
    int phases;        // deterministic: bit 0 preprocess, bit 1 dK/dV kernel, bit 2 dQ kernel;
                       // single pass: bit 3 preprocess + zero dQ accumulator, bit 4 fused
                       // dK/dV/dQ kernel, bit 5 dQ accumulator -> bf16
    int num_sms;       // persistent grid size
};

cudaError_t launch_fwd(const FwdLaunch &a, cudaStream_t stream);
cudaError_t launch_fwd_fp8(const FwdLaunch &a, cudaStream_t stream);  // tm_q/tm_k/tm_v: e4m3 maps
cudaError_t launch_bwd(const BwdLaunch &a, cudaStream_t stream);
// the backward's per-row terms D and lse2 (and, with zero_dqacc, zeroes a.dqacc)
cudaError_t launch_bwd_pre(const BwdLaunch &a, bool zero_dqacc, cudaStream_t stream);
cudaError_t launch_bwd_fused(const BwdLaunch &a, cudaStream_t stream);  // phases bits 3-5
// A zeroed {units claimed, CTAs finished} counter pair in device memory for one launch
// of a kernel with a dynamic unit deal (null if the device's pool cannot be reached).
unsigned int *next_sched_slot();
// Slices per band forced by attn_debug_force_band (0: the launchers choose).
int forced_band();

}  // namespace attn
