// Sigmoid top-k selection of one token, shared by the prefill router GEMM
// epilogue (TopK), the split-K router reduction and the decode routing
// kernel (warp_topk_regs / warp_topk) so all paths take identical decisions
// in float32.
//
// NemotronMoeLayer (nemotron_moe.rs module documentation): sigmoid top-k
// routing.  Selection key = sigmoid(logit) + bias (bias for selection only);
// slots are kept in descending key order and a key only displaces strictly
// smaller ones, so on equal keys the lower expert index (visited first) wins.
// Weights: the unbiased scores of the selected experts renormalised to sum 1
// and multiplied by routed_scaling_factor.
#pragma once

namespace moe {

constexpr int kTopKMax = 16;

struct TopK {
  float key[kTopKMax];
  float score[kTopKMax];
  int id[kTopKMax];

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < kTopKMax; ++j) {
      key[j] = -INFINITY;
      score[j] = 0.f;
      id[j] = -1;
    }
  }

  // Offer expert e (experts must be offered in increasing index order).
  __device__ __forceinline__ void offer(int e, float logit, float bias, int k) {
    const float s = 1.0f / (1.0f + expf(-logit));
    const float kk = s + bias;
#pragma unroll
    for (int x = kTopKMax - 1; x >= 0; --x) {
      if (x < k && kk > key[x]) {
        if (x > 0 && kk > key[x - 1]) {
          key[x] = key[x - 1];
          score[x] = score[x - 1];
          id[x] = id[x - 1];
        } else {
          key[x] = kk;
          score[x] = s;
          id[x] = e;
        }
      }
    }
  }

  // Renormalised weights times rsf into w[0..k), ids into idx[0..k).
  __device__ __forceinline__ void write(int k, float rsf, int* idx, float* w) const {
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kTopKMax; ++j)
      if (j < k) sum += score[j];
    const float scale = rsf / sum;
#pragma unroll
    for (int j = 0; j < kTopKMax; ++j) {
      if (j < k) {
        idx[j] = id[j];
        w[j] = score[j] * scale;
      }
    }
  }
};

// Order-preserving bits of a selection key: for keys a, b that are not NaN,
// a > b exactly when key_bits(a) > key_bits(b) as unsigned integers (-0 is
// taken as +0).  NaN maps to 0, below every other key (a NaN key is never
// chosen: no comparison with it is true); -inf maps to kKeyNegInf.
constexpr uint32_t kKeyNegInf = 0x007FFFFFu;
__device__ __forceinline__ uint32_t key_bits(float f) {
  if (f != f) return 0u;
  const uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp-cooperative top-k of one token's E <= 256 logits (same selection rule
// and weight formula as TopK): lane l holds the logits of experts l, l + 32,
// ... in lg[].  k rounds of a warp arg-max on (key descending, expert index
// ascending): a warp-wide integer max of the key bits, then a warp-wide min
// of the expert indices that hold that key.  A round in which no remaining
// key beats -inf (only with NaN or infinite inputs) chooses id 0x7fffffff,
// as a plain scan from -inf would.  idx[0..k) and w[0..k) are written by the
// warp (global or shared memory).  Returns, on lanes < k, the expert chosen
// in round `lane` (-1 elsewhere).
__device__ __forceinline__ int warp_topk_regs(const float (&lg)[8], const float* bias, int E,
                                              int k, float rsf, int* idx, float* w) {
  const int lane = threadIdx.x & 31;
  uint32_t key[8];
  float sc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    if (e < E) {
      const float s = 1.0f / (1.0f + expf(-lg[j]));
      sc[j] = s;
      key[j] = key_bits(s + (bias ? bias[e] : 0.0f));
    } else {
      sc[j] = 0.f;
      key[j] = kKeyNegInf;
    }
  }
  float sum = 0.f, mine = 0.f;
  int mine_e = -1;
  for (int r = 0; r < k; ++r) {
    uint32_t lm = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) lm = key[j] > lm ? key[j] : lm;
    const uint32_t m = __reduce_max_sync(0xffffffffu, lm);
    int be = 0x7fffffff;
    if (m > kKeyNegInf) {
      int mi = 0x7fffffff;
#pragma unroll
      for (int j = 7; j >= 0; --j)
        if (key[j] == m) mi = lane + 32 * j;
      be = __reduce_min_sync(0xffffffffu, mi);
    }
    float s = 0.f;
    if ((be & 31) == lane) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (lane + 32 * j == be) {
          s = sc[j];
          key[j] = 0u;
        }
      }
    }
    s = __shfl_sync(0xffffffffu, s, be & 31);
    sum += s;
    if (lane == r) {
      mine = s;
      mine_e = be;
      idx[r] = be;
    }
  }
  if (lane < k) w[lane] = mine * (rsf / sum);
  return mine_e;
}

// Same, reading the logits from global memory (logits[0..E)).
__device__ __forceinline__ void warp_topk(const float* logits, const float* bias, int E, int k,
                                          float rsf, int* idx, float* w) {
  const int lane = threadIdx.x & 31;
  float lg[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) lg[j] = lane + 32 * j < E ? __ldcg(logits + lane + 32 * j) : 0.f;
  warp_topk_regs(lg, bias, E, k, rsf, idx, w);
}

}  // namespace moe
