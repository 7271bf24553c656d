// Small-batch decode path (1 <= T <= 8): the layer is weight-streaming at
// these sizes (NemotronMoeLayer `decode`; MoeLayer `forward_k2`/`forward_k3`
// batch a few tokens through one weight sweep).  Three launches:
//   decode_route (CUDA cores): RMSNorm, FP32 router logits, sigmoid top-k,
//       the distinct-expert segment table and the tile lists of the next two
//       launches.
//   grouped GEMM, up (tcgen05, weights x tokens, N = 16): relu^2 of every
//       distinct routed expert's up rows and of the shared expert's.
//   grouped GEMM, down: a 128-row block of the output accumulates the
//       shared expert's and every routed slot's k-blocks in one pass
//       (concatenated K); the last piece of the block to finish adds the
//       pieces in k order and the residual into hidden.
// Both GEMM launches cut their k-blocks into equal contiguous ranges, one
// per CTA (stream-K), so every SM streams the same number of weight bytes.
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
  __nv_bfloat16* ub;       // [(Umax + 1) * 16, I] w_t * relu^2(up) per segment, token-major
  __nv_bfloat16* vb;       // [16, S] shared relu^2(up), token-major
  float* up_part;          // [up tiles + CTAs, 128, 16] up piece partials
  unsigned* up_counter;    // [up tiles] pieces finished per tile (self-resetting)
  float* partial;          // [ceil(H/128) + CTAs, 128, 16] down piece partials
  unsigned* mt_counter;    // [ceil(H/128)] pieces finished per row tile (self-resetting)
};

inline int decode_max_slots(const moe_config& c) {
  const int p = kDecodeMaxT * c.top_k;
  return p < c.num_experts ? p : c.num_experts;
}

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// ctas: grid of the decode GEMM launches (one CTA per SM).
template <class Take>
void carve_decode(DecodeWorkspace* d, const moe_config& c, int ctas, Take take) {
  const size_t k = c.top_k, E = c.num_experts, H = c.hidden_size, I = c.moe_inter,
               S = c.shared_inter;
  const size_t U = decode_max_slots(c);
  const size_t up_tiles = U * cdiv(int(I), kBM) + cdiv(int(S), kBM);
  const size_t down_tiles = cdiv(int(H), kBM);
  d->x16 = reinterpret_cast<__nv_bfloat16*>(take(kDecodeN * H * 2));
  d->logits = reinterpret_cast<float*>(take(kDecodeMaxT * E * 4));
  d->idx = reinterpret_cast<int*>(take(kDecodeMaxT * k * 4));
  d->w = reinterpret_cast<float*>(take(kDecodeMaxT * k * 4));
  d->seg_expert = reinterpret_cast<int*>(take((U + 1) * 4));
  d->seg_w = reinterpret_cast<float*>(take((U + 1) * kDecodeN * 4));
  d->n_segments = reinterpret_cast<int*>(take(4));
  d->counter = reinterpret_cast<unsigned*>(take(4));
  d->tiles_up = reinterpret_cast<DecodeTile*>(take(up_tiles * sizeof(DecodeTile)));
  d->n_tiles_up = reinterpret_cast<int*>(take(4));
  d->ub = reinterpret_cast<__nv_bfloat16*>(take((U + 1) * kDecodeN * I * 2));
  d->vb = reinterpret_cast<__nv_bfloat16*>(take(kDecodeN * S * 2));
  d->up_part = reinterpret_cast<float*>(take((up_tiles + ctas) * kBM * kDecodeN * 4));
  d->up_counter = reinterpret_cast<unsigned*>(take(up_tiles * 4));
  d->partial = reinterpret_cast<float*>(take((down_tiles + ctas) * kBM * kDecodeN * 4));
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
