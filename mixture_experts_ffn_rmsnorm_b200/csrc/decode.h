// Small-batch decode path (1 <= T <= 8): the layer is weight-streaming at
// these sizes (NemotronMoeLayer `decode`; MoeLayer `forward_k2`/`forward_k3`
// batch a few tokens through one weight sweep).  Three launches:
//   decode_route (CUDA cores): RMSNorm, FP32 router logits, sigmoid top-k,
//       the distinct-expert segment table and the tile lists of the next two
//       launches.
//   grouped GEMM, up (tcgen05, weights x tokens, N = 16): relu^2 of every
//       distinct routed expert's up rows and of the shared expert's.
//   grouped GEMM, down (split by segment): every segment's down rows; the last
//       segment of a 128-row tile to finish sums all segments in a fixed order
//       with the residual into hidden.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace moe {

constexpr int kDecodeMaxT = MOE_DECODE_MAX_TOKENS;
constexpr int kDecodeN = 16;  // token columns of a decode tile (UMMA N)

struct DecodeWorkspace {
  __nv_bfloat16* x16;      // [16, H]  bf16(n) of the tokens (rows >= T unused)
  float* logits;           // [8, E]
  int* idx;                // [8, k]
  float* w;                // [8, k]
  int* seg_expert;         // [Umax + 1] expert of segment s >= 1 (segment 0 = shared)
  float* seg_w;            // [Umax + 1, 16] routing weight of token t in segment s (0 = not routed)
  int* n_segments;         // [1] 1 + distinct experts
  unsigned* counter;       // [1] router blocks finished (self-resetting)
  DecodeTile* tiles_up;    // [Umax * ceil(I/128) + ceil(S/128)]
  int* n_tiles_up;         // [1]
  DecodeTile* tiles_down;  // [(Umax + 1) * ceil(H/128)]
  int* n_tiles_down;       // [1]
  __nv_bfloat16* ub;       // [(Umax + 1) * 16, I] w_t * relu^2(up) per segment, token-major
  __nv_bfloat16* vb;       // [16, S] shared relu^2(up), token-major
  float* partial;          // [(Umax + 1), H, 16] down output per segment
  unsigned* mt_counter;    // [ceil(H/128)] segments finished per row tile (self-resetting)
};

inline int decode_max_slots(const moe_config& c) {
  const int p = kDecodeMaxT * c.top_k;
  return p < c.num_experts ? p : c.num_experts;
}

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

template <class Take>
void carve_decode(DecodeWorkspace* d, const moe_config& c, Take take) {
  const size_t k = c.top_k, E = c.num_experts, H = c.hidden_size, I = c.moe_inter,
               S = c.shared_inter;
  const size_t U = decode_max_slots(c);
  d->x16 = reinterpret_cast<__nv_bfloat16*>(take(kDecodeN * H * 2));
  d->logits = reinterpret_cast<float*>(take(kDecodeMaxT * E * 4));
  d->idx = reinterpret_cast<int*>(take(kDecodeMaxT * k * 4));
  d->w = reinterpret_cast<float*>(take(kDecodeMaxT * k * 4));
  d->seg_expert = reinterpret_cast<int*>(take((U + 1) * 4));
  d->seg_w = reinterpret_cast<float*>(take((U + 1) * kDecodeN * 4));
  d->n_segments = reinterpret_cast<int*>(take(4));
  d->counter = reinterpret_cast<unsigned*>(take(4));
  d->tiles_up = reinterpret_cast<DecodeTile*>(
      take((U * cdiv(int(I), kBM) + cdiv(int(S), kBM)) * sizeof(DecodeTile)));
  d->n_tiles_up = reinterpret_cast<int*>(take(4));
  d->tiles_down =
      reinterpret_cast<DecodeTile*>(take((U + 1) * cdiv(int(H), kBM) * sizeof(DecodeTile)));
  d->n_tiles_down = reinterpret_cast<int*>(take(4));
  d->ub = reinterpret_cast<__nv_bfloat16*>(take((U + 1) * kDecodeN * I * 2));
  d->vb = reinterpret_cast<__nv_bfloat16*>(take(kDecodeN * S * 2));
  d->partial = reinterpret_cast<float*>(take((U + 1) * H * kDecodeN * 4));
  d->mt_counter = reinterpret_cast<unsigned*>(take(cdiv(int(H), kBM) * 4));
}

struct DecodeRouteArgs {
  const moe_config* cfg;
  const moe_weights* w;
  const DecodeWorkspace* ws;
  const __nv_bfloat16* hidden;
  __nv_bfloat16* residual;
  int T;
};

// Whether the decode path covers this configuration (direct layer, BF16
// experts, the router rows fit the kernel's shared memory).
bool decode_supported(const moe_config& c);
cudaError_t prepare_decode();
cudaError_t launch_decode_route(const DecodeRouteArgs& a, cudaStream_t stream);

}  // namespace moe
