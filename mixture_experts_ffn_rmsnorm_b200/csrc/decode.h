// Small-batch decode path (1 <= T <= 8): the layer is weight-streaming at
// these sizes (NemotronMoeLayer `decode`; MoeLayer `forward_k2`/`forward_k3`
// batch a few tokens through one weight sweep).  One cooperative launch
// (decode_fused.cu) does the RMSNorm, the FP32 router, the sigmoid top-k,
// the shared and routed up projections with relu^2 and the down projections
// with the weighted sum and the residual add, with the weights as the
// 128-row tcgen05 operand and the tokens as N = 16.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace moe {

constexpr int kDecodeMaxT = MOE_DECODE_MAX_TOKENS;
constexpr int kDecodeN = 16;  // token columns of a decode tile (UMMA N)

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Workspace of the single-launch decode path (decode_fused.cu).  The
// synchronisation words, the accumulator and the marks start at zero (the
// workspace is cleared at creation) and every launch leaves them at zero:
// each CTA clears the accumulator rows it finishes, and the last CTA to exit
// resets the synchronisation words.
struct FusedWorkspace {
  __nv_bfloat16* x16;      // [CTAs, 16, H] each CTA's copy of bf16(n) of the tokens (rows >= T unused)
  uint8_t* x8;             // [CTAs, 16, H] E4M3 copy of x * w (one-token FP8 launch, W8A8; row 0 used)
  float* logits;           // [8, E]
  int* idx;                // [8, k] routing of the pass (for moe_copy_routing)
  float* w;                // [8, k]
  long long* acc;          // [8, H] fixed-point sum of the CTAs' partial outputs (token-major)
  uint8_t* bad;            // [8, H] 1 where a partial was not finite or out of range
  unsigned* sync;          // [4] logit arrivals, partial outputs added, exited CTAs
};

// ctas: grid of the decode launch (one CTA per SM).
template <class Take>
void carve_fused(FusedWorkspace* d, const moe_config& c, int ctas, Take take) {
  const size_t k = c.top_k, E = c.num_experts, H = c.hidden_size;
  d->x16 = reinterpret_cast<__nv_bfloat16*>(take(size_t(ctas) * kDecodeN * H * 2));
  d->x8 = reinterpret_cast<uint8_t*>(take(size_t(ctas) * kDecodeN * H));
  d->logits = reinterpret_cast<float*>(take(kDecodeMaxT * E * 4));
  d->idx = reinterpret_cast<int*>(take(kDecodeMaxT * k * 4));
  d->w = reinterpret_cast<float*>(take(kDecodeMaxT * k * 4));
  d->acc = reinterpret_cast<long long*>(take(kDecodeMaxT * H * 8));
  d->bad = reinterpret_cast<uint8_t*>(take(kDecodeMaxT * H));
  d->sync = reinterpret_cast<unsigned*>(take(4 * 4));
}

struct FusedDecodeArgs {
  const moe_config* cfg;
  const moe_weights* w;
  const FusedWorkspace* ws;
  const CUtensorMap *tm_up, *tm_sup, *tm_down, *tm_sdown;  // weights as 128-row A boxes
  const CUtensorMap *tm_up64, *tm_sup64;  // up weights as 64-row A boxes (units of 64 rows)
  const CUtensorMap* tm_x[4];  // token rows, B boxes of 1, 2, 4, 8 rows (token-count bucket)
  const CUtensorMap* tm_x8;    // E4M3 token rows (x8), boxes of one row x 128 bytes
  __nv_bfloat16* hidden;    // [T, H] input rows
  __nv_bfloat16* residual;  // [T, H] written with the input rows (device or mapped host memory)
  __nv_bfloat16* out;       // [T, H] output rows (device or mapped host memory); null: hidden
  int T;
  int grid;
  int* status;
};

// Whether the single-launch decode path covers this configuration (direct
// layer, BF16 routed and shared experts) on a grid of `grid` CTAs.
bool fused_decode_supported(const moe_config& c, int grid);
cudaError_t prepare_fused_decode();
cudaError_t launch_fused_decode(const FusedDecodeArgs& a, cudaStream_t stream);

}  // namespace moe
