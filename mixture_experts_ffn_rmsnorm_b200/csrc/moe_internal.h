// Internal declarations shared by the kernels and the C-ABI host code.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kBM = 128;             // GEMM tile rows (UMMA M)
constexpr int kGemmThreads = 192;    // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kMaxTopKShared = 16;   // top_k bound of the routing kernels

// What the GEMM epilogue does with an accumulator row segment.
enum EpiKind : int {
  EPI_BF16 = 0,        // out = bf16(acc)
  EPI_RELU2_BF16 = 1,  // out = bf16(max(acc, 0)^2)
  EPI_F32 = 2,         // out = acc (float32)
  EPI_TOPK = 3,        // sigmoid top-k routing of the row (gate logits never stored)
  EPI_BLEND = 4,       // out = bf16(acc + blend_s + blend_res)  (LatentMoE fc2)
};

// Counts the kernels a call enqueues and, when profiling is enabled, records
// caller-owned CUDA events around them: events[0] before the first launch,
// events[i] after the i-th.
// While the stream is being captured into a CUDA graph the events are
// recorded as external event nodes, so they time every replay.
struct LaunchLog {
  int count = 0;
  void* const* events = nullptr;
  int nevents = 0;
  unsigned flags = cudaEventRecordDefault;
  void record(int i, cudaStream_t s) const {
    cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), s, flags);
  }
  void begin(cudaStream_t s) {
    if (nevents <= 0) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
      flags = cudaEventRecordExternal;
    record(0, s);
  }
  void done(cudaStream_t s) {
    ++count;
    if (count < nevents) record(count, s);
  }
};

// One class of GEMM tiles inside a launch.  A is [rows, K] (K contiguous),
// B is [groups * N, K]; a tile multiplies 128 rows of A by BN rows of one
// group of B.
struct GemmClass {
  int K;                  // reduction length in elements
  int N;                  // output columns of one group (B rows per group)
  int ntiles;             // ceil(N / BN)
  int mtiles;             // m-tiles of a dense class (ignored when the launch has a tile table)
  int rows;               // valid A rows of a dense class
  int a_kwrap;            // A's k coordinate is taken modulo this (0 = no wrap)
  int b_kwrap;            // B's k coordinate is taken modulo this (0 = no wrap)
  int ksplit;             // dense classes: K-block ranges per output tile (0 or 1 = whole K)
  int epi;                // EpiKind
  void* out;              // output base
  int ldo;                // output row stride in elements
  const float* col_scale; // [groups, N] per-output-column scale (FP8 weights) or null
  const float* row_scale; // [rows] per-A-row scale or null
  int fp8;                // operands are E4M3 (kind::f8f6f4, 128 K elements per stage)
  unsigned* row_amax;     // per output row max (float bits, values >= 0) or null
};

struct GemmParams {
  CUtensorMap tmA[2];
  CUtensorMap tmB[2];
  GemmClass cls[2];
  int nclasses;
  // Grouped class 0: m-tile i covers sorted rows [tile_table[i].y, +128)
  // of group tile_table[i].x; rows at or beyond group_off[x + 1] belong to the
  // next group and are not stored.  n_mtiles is the device-side tile count.
  const int2* tile_table;
  const int* n_mtiles;
  const int* group_off;
  // EPI_TOPK
  const float* gate_bias;
  int top_k;
  int num_experts;
  float rsf;
  int* topk_idx;
  float* topk_w;
  const float* topk_rs;    // per-row factor of the logits (the token's RMSNorm factor) or null
  float* topk_part;        // split-K partial logits [ksplit][topk_rows_cap][E]
  int topk_rows_cap;
  int* expert_hist;        // [token tiles][E] experts chosen by each 128-token tile
  // EPI_BLEND
  const float* blend_s;
  const __nv_bfloat16* blend_res;
  int* status;
  // Only the epilogue warps wait for the previous launch (griddepcontrol):
  // the operands the producer loads do not depend on it, only what the
  // epilogue reads does (the router: the RMSNorm factors).
  int epi_wait;
  // Dynamic tile schedule (null = static round-robin):
  // sched[0] hands out tile indices past the first gridDim.x, sched[1]
  // counts exiting CTAs.  Both are zero before the launch and the last CTA
  // to exit zeroes them again.  Tiles are then taken shared class first
  // (its tiles have the longer K), routed class after.
  int* sched;
};

// Launch the persistent grouped GEMM (bn = 128 or 256); the operand type
// is a per-class property (GemmClass::fp8).  pdl: launch with programmatic
// stream serialization (the kernel waits on griddepcontrol before reading
// anything the previous kernel wrote).
cudaError_t launch_grouped_gemm(const GemmParams& p, int bn, int grid, cudaStream_t stream,
                                bool pdl = false);
// Set the dynamic shared memory limit of every GEMM instantiation on the
// current device (call once per device before launching).
cudaError_t prepare_grouped_gemm();

// Routing / sort / data movement kernels (route.cu).
// RMSNorm: residual <- hidden, rs[t] = rsqrt(mean x^2 + eps), bf16 normed
// rows into the first H columns of gate_a [T, 2H].
// normed_q/normed_scale (nullable): per-token E4M3 copy of the normed rows.
// hist_clear[0..n_clear) is zeroed on the way (the split-K router's
// histogram, accumulated with atomics); may be null.
cudaError_t launch_rmsnorm(const __nv_bfloat16* hidden, const __nv_bfloat16* norm_w,
                           __nv_bfloat16* residual, __nv_bfloat16* gate_a, float* rs,
                           uint8_t* normed_q, float* normed_scale, int T, int H, float eps,
                           int* hist_clear, int n_clear, cudaStream_t stream);
// The router's gate with the norm weight folded in: out [E, 2H] =
// [bf16(G * w) | bf16(G * w - bf16(G * w))] (fp32 products), once per layer.
cudaError_t launch_prep_gate(const __nv_bfloat16* gate, const __nv_bfloat16* norm_w, int E, int H,
                             __nv_bfloat16* out, cudaStream_t stream);
// Split-K router, second half: logits = rs[t] * the sum of the ks partials
// in split order, sigmoid top-k per token into idx/w, and hist[t / 128][e]
// += 1 for every chosen expert (hist zeroed beforehand).  Launched as a
// programmatic dependent of the router GEMM.
constexpr int kRouterMaxSplit = 16;
cudaError_t launch_router_reduce(const float* part, int ks, int rows_cap, int T, int E,
                                 const float* bias, int k, float rsf, const float* rs, int* idx,
                                 float* w, int* hist, cudaStream_t stream);
// Stable sort by expert from the routing table idx [T, k] and its per-128-
// token-tile expert histogram hist [ceil(T/128), E].
cudaError_t launch_tile_hist(const int* idx, int T, int k, int E, int* hist, int* status,
                             cudaStream_t stream);
cudaError_t launch_sort(const int* idx, const int* hist, int T, int k, int E, int* perm, int* inv,
                        int* off, int2* tile_table, int* n_mtiles, int* status,
                        cudaStream_t stream);
// Row gather: xs[p] = X[perm[p] / k] (row_bytes per row; ldx_bytes source
// stride); optionally scales: xs_scale[p] = scale[perm[p] / k].
cudaError_t launch_gather(const void* X, size_t ldx_bytes, const int* perm, int k, int R,
                          int row_bytes, void* xs, const float* scale, float* xs_scale,
                          cudaStream_t stream);
// Per-row E4M3 quantisation of u [R, I] and v [Rv, S] (bf16) with their
// row maxima (float bits, reset to 0 afterwards): q = sat(x / s),
// s = amax / 448.  One launch for both sets (either may be empty).
cudaError_t launch_quantize_rows(const __nv_bfloat16* u, unsigned* u_amax, uint8_t* uq,
                                 float* u_scale, int R, int I, const __nv_bfloat16* v,
                                 unsigned* v_amax, uint8_t* vq, float* v_scale, int Rv, int S,
                                 cudaStream_t stream);
cudaError_t launch_combine(const __nv_bfloat16* y, const int* inv, const float* w,
                           const float* s, const __nv_bfloat16* residual,
                           __nv_bfloat16* hidden, int T, int k, int H, cudaStream_t stream);
// mq / m_scale (nullable): the E4M3 copy of m with one scale per row.
cudaError_t launch_latent_reduce(const __nv_bfloat16* y, const int* inv, const float* w,
                                 __nv_bfloat16* m, uint8_t* mq, float* m_scale, int T, int k,
                                 int L, cudaStream_t stream);

}  // namespace moe
