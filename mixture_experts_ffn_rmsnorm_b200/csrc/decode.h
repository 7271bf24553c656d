// Small-batch decode path (1 <= T <= 8): the layer is weight-streaming at
// these sizes, so it runs as bandwidth-bound GEMVs that read each distinct
// routed expert's weights once for all tokens routed to it, plus the shared
// expert's weights once (NemotronMoeLayer `decode`; MoeLayer `forward_k2` /
// `forward_k3` for the batched small-T idea).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace moe {

constexpr int kDecodeMaxT = MOE_DECODE_MAX_TOKENS;

struct DecodeWorkspace {
  __nv_bfloat16* normed;   // [8, H]  bf16(n), the experts' input
  float* logits;           // [8, E]
  int* idx;                // [8, k]
  float* w;                // [8, k]
  int* slot_expert;        // [Umax] distinct routed experts, first-use order
  int* slot_cnt;           // [Umax] tokens routed to the slot
  int* slot_tok;           // [Umax, 8] token of the slot's j-th pair
  int* slot_pair;          // [Umax, 8] flat pair index t*k + j
  float* slot_w;           // [Umax, 8] routing weight of the pair
  int* n_slots;            // [1]
  unsigned* counter;       // [1] router blocks finished (self-resetting)
  __nv_bfloat16* uo;       // [8*k, I] relu^2(up) per (token, slot) pair
  __nv_bfloat16* vo;       // [8, S]   shared relu^2(up)
  float* sh;               // [8, H]   shared down output
};

inline int decode_max_slots(const moe_config& c) {
  const int p = kDecodeMaxT * c.top_k;
  return p < c.num_experts ? p : c.num_experts;
}

template <class Take>
void carve_decode(DecodeWorkspace* d, const moe_config& c, Take take) {
  const size_t T = kDecodeMaxT, k = c.top_k, E = c.num_experts, H = c.hidden_size;
  const size_t U = decode_max_slots(c);
  d->normed = reinterpret_cast<__nv_bfloat16*>(take(T * H * 2));
  d->logits = reinterpret_cast<float*>(take(T * E * 4));
  d->idx = reinterpret_cast<int*>(take(T * k * 4));
  d->w = reinterpret_cast<float*>(take(T * k * 4));
  d->slot_expert = reinterpret_cast<int*>(take(U * 4));
  d->slot_cnt = reinterpret_cast<int*>(take(U * 4));
  d->slot_tok = reinterpret_cast<int*>(take(U * T * 4));
  d->slot_pair = reinterpret_cast<int*>(take(U * T * 4));
  d->slot_w = reinterpret_cast<float*>(take(U * T * 4));
  d->n_slots = reinterpret_cast<int*>(take(4));
  d->counter = reinterpret_cast<unsigned*>(take(4));
  d->uo = reinterpret_cast<__nv_bfloat16*>(take(T * k * c.moe_inter * 2));
  d->vo = reinterpret_cast<__nv_bfloat16*>(take(T * c.shared_inter * 2));
  d->sh = reinterpret_cast<float*>(take(T * H * 4));
}

struct DecodeArgs {
  const moe_config* cfg;
  const moe_weights* w;
  const DecodeWorkspace* ws;
  int* status;
  int num_sms;
};

// Whether the decode kernels cover this configuration (direct layer with
// BF16 experts, at most MOE_MAX_EXPERTS experts).
bool decode_supported(const moe_config& c);
cudaError_t prepare_decode();
moe_status enqueue_decode(const DecodeArgs& a, __nv_bfloat16* hidden, __nv_bfloat16* residual,
                          int T, cudaStream_t stream, LaunchLog* log);

}  // namespace moe
