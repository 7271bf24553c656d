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

// Warp-cooperative top-k of one token's E <= 256 logits (same selection rule
// and weight formula as TopK): lane l holds the logits of experts l, l + 32,
// ... in lg[]; k rounds of a warp arg-max on (key descending, expert index
// ascending).  idx[0..k) and w[0..k) are written by the warp (global or
// shared memory).  Returns, on lanes < k, the expert chosen in round `lane`
// (-1 elsewhere).
__device__ __forceinline__ int warp_topk_regs(const float (&lg)[8], const float* bias, int E,
                                              int k, float rsf, int* idx, float* w) {
  const int lane = threadIdx.x & 31;
  float key[8], sc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    if (e < E) {
      const float s = 1.0f / (1.0f + expf(-lg[j]));
      sc[j] = s;
      key[j] = s + (bias ? bias[e] : 0.0f);
    } else {
      sc[j] = 0.f;
      key[j] = -INFINITY;
    }
  }
  float sum = 0.f, mine = 0.f;
  int mine_e = -1;
  for (int r = 0; r < k; ++r) {
    float bk = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (key[j] > bk) {
        bk = key[j];
        be = lane + 32 * j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
      }
    }
    float s = 0.f;
    if ((be & 31) == lane) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (lane + 32 * j == be) {
          s = sc[j];
          key[j] = -INFINITY;
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
