// Decode path kernels (1 <= T <= 8 tokens).
//
//   decode_route_shared_up: blocks [0, G) compute RMSNorm + FP32 router
//       logits (one warp per expert row); the last of them to finish runs the
//       sigmoid top-k for every token and builds the distinct-expert slot
//       list.  Blocks [G, G + S/32) compute the shared expert's up projection
//       + relu^2 meanwhile (it does not depend on routing).
//   decode_up:    one block per (routed slot, 32 rows of I): up + relu^2 for
//                 the tokens routed to that expert, weights read once.
//   decode_down:  one block per (slot, 32 rows of H): down projection per
//                 routed (token, slot) pair; the extra slot is the shared
//                 expert's down projection.
//   decode_combine: hidden = residual + shared + sum_j w_j * y_j.
// All GEMVs stream weight rows with 16-byte loads, 4 rows per warp, and take
// the token vectors from shared memory.
#include "decode.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerBlock = kWarps * kRowsPerWarp;  // 32

__device__ __forceinline__ float lo16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  f[0] = lo16(u.x); f[1] = hi16(u.x);
  f[2] = lo16(u.y); f[3] = hi16(u.y);
  f[4] = lo16(u.z); f[5] = hi16(u.z);
  f[6] = lo16(u.w); f[7] = hi16(u.w);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// acc[r][t] = sum_i W[r][i] * X[t][i] for NT token rows X (bf16, shared
// memory, row stride K) and kRowsPerWarp weight rows starting at W (global,
// row stride ldw).  Rows at or beyond nrows are skipped.  Result valid in
// every lane after the warp reduction.
template <int NT>
__device__ __forceinline__ void warp_gemv(const bf16* __restrict__ W, size_t ldw, int nrows,
                                          int K, const bf16* xs,
                                          float (&acc)[kRowsPerWarp][NT]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[r][t] = 0.f;
  for (int i = lane * 8; i < K; i += 256) {
    uint4 wv[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
      wv[r] = r < nrows ? __ldcs(reinterpret_cast<const uint4*>(W + r * ldw + i))
                        : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float x[8];
      unpack8(*reinterpret_cast<const uint4*>(xs + t * K + i), x);
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        float g[8];
        unpack8(wv[r], g);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[r][t] = fmaf(g[q], x[q], acc[r][t]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[r][t] = warp_sum(acc[r][t]);
}

// Copy token rows into shared memory (bf16, K contiguous per row).
__device__ __forceinline__ void stage_rows(bf16* xs, const bf16* const* src, int n, int K) {
  const int nv = K / 8;
  for (int i = threadIdx.x; i < n * nv; i += kThreads) {
    const int t = i / nv, c = i - t * nv;
    reinterpret_cast<uint4*>(xs + t * K)[c] = reinterpret_cast<const uint4*>(src[t])[c];
  }
}

__device__ __forceinline__ float relu2(float x) { return x > 0.f ? x * x : 0.f; }

// Up projection (+ relu^2) of 32 rows for NT tokens, written as bf16.
// out[t] points at token t's output row; column c = row0 + local row.
template <int NT>
__device__ void up_rows(const bf16* W, int K, int nrows_total, int row0, const bf16* xs,
                        bf16* const* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = row0 + warp * kRowsPerWarp;
  if (r0 >= nrows_total) return;
  float acc[kRowsPerWarp][NT];
  warp_gemv<NT>(W + size_t(r0) * K, K, nrows_total - r0, K, xs, acc);
  if (lane < kRowsPerWarp * NT) {
    const int r = lane / NT, t = lane - r * NT;
    float v = 0.f;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr)
#pragma unroll
      for (int tt = 0; tt < NT; ++tt)
        if (rr == r && tt == t) v = acc[rr][tt];
    if (r0 + r < nrows_total) out[t][r0 + r] = __float2bfloat16_rn(relu2(v));
  }
}

// Down projection of 32 rows for NT tokens, float32, unscaled.
template <int NT>
__device__ void down_rows(const bf16* W, int K, int nrows_total, int row0, const bf16* xs,
                          float* const* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = row0 + warp * kRowsPerWarp;
  if (r0 >= nrows_total) return;
  float acc[kRowsPerWarp][NT];
  warp_gemv<NT>(W + size_t(r0) * K, K, nrows_total - r0, K, xs, acc);
  if (lane < kRowsPerWarp * NT) {
    const int r = lane / NT, t = lane - r * NT;
    float v = 0.f;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr)
#pragma unroll
      for (int tt = 0; tt < NT; ++tt)
        if (rr == r && tt == t) v = acc[rr][tt];
    if (r0 + r < nrows_total) out[t][r0 + r] = v;
  }
}

#define MOE_DISPATCH_NT(n, CALL)  \
  switch (n) {                    \
    case 1: { constexpr int NT = 1; CALL; } break; \
    case 2: { constexpr int NT = 2; CALL; } break; \
    case 3: { constexpr int NT = 3; CALL; } break; \
    case 4: { constexpr int NT = 4; CALL; } break; \
    case 5: { constexpr int NT = 5; CALL; } break; \
    case 6: { constexpr int NT = 6; CALL; } break; \
    case 7: { constexpr int NT = 7; CALL; } break; \
    case 8: { constexpr int NT = 8; CALL; } break; \
    default: break;               \
  }

struct RouteParams {
  const bf16* hidden;
  const bf16* norm_w;
  const bf16* gate_w;
  const float* gate_bias;
  const bf16* shared_up_w;
  bf16* residual;
  DecodeWorkspace ws;
  int T, H, E, k, S, umax, gate_blocks;
  float eps, rsf;
};

__global__ void __launch_bounds__(kThreads) decode_route_shared_up(const RouteParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float rs[kDecodeMaxT];
  __shared__ int am_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.H, T = p.T;

  // RMSNorm scale of every token (each block recomputes it; rows are tiny).
  for (int t = warp; t < T; t += kWarps) {
    const uint4* x = reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H);
    float ss = 0.f;
    for (int i = lane; i < H / 8; i += 32) {
      float f[8];
      unpack8(x[i], f);
#pragma unroll
      for (int q = 0; q < 8; ++q) ss += f[q] * f[q];
    }
    ss = warp_sum(ss);
    if (lane == 0) rs[t] = rsqrtf(ss / float(H) + p.eps);
  }
  __syncthreads();

  if (blockIdx.x >= p.gate_blocks) {
    // ---- shared expert up projection + relu^2 on bf16(n)
    bf16* xs = reinterpret_cast<bf16*>(dsm);
    const int nv = H / 8;
    for (int i = threadIdx.x; i < T * nv; i += kThreads) {
      const int t = i / nv, c = i - t * nv;
      float f[8], g[8];
      unpack8(reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[c], f);
      unpack8(reinterpret_cast<const uint4*>(p.norm_w)[c], g);
      bf16* d = xs + t * H + c * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) d[q] = __float2bfloat16_rn(f[q] * rs[t] * g[q]);
    }
    __syncthreads();
    bf16* outs[kDecodeMaxT];
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) outs[t] = p.ws.vo + size_t(t) * p.S;
    const int row0 = (blockIdx.x - p.gate_blocks) * kRowsPerBlock;
    MOE_DISPATCH_NT(T, (up_rows<NT>(p.shared_up_w, H, p.S, row0, xs, outs)));
    return;
  }

  // ---- router logits in float32 from the un-rounded normed vector
  float* xn = reinterpret_cast<float*>(dsm);  // [T][H]
  const int nv = H / 8;
  for (int i = threadIdx.x; i < T * nv; i += kThreads) {
    const int t = i / nv, c = i - t * nv;
    const uint4 hv = reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[c];
    float f[8], g[8];
    unpack8(hv, f);
    unpack8(reinterpret_cast<const uint4*>(p.norm_w)[c], g);
    float* d = xn + t * H + c * 8;
#pragma unroll
    for (int q = 0; q < 8; ++q) d[q] = f[q] * rs[t] * g[q];
    if (blockIdx.x == 0) {
      reinterpret_cast<uint4*>(p.residual + size_t(t) * H)[c] = hv;
      bf16* nb = p.ws.normed + size_t(t) * H + c * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) nb[q] = __float2bfloat16_rn(d[q]);
    }
  }
  __syncthreads();
  for (int e = blockIdx.x * kWarps + warp; e < p.E; e += p.gate_blocks * kWarps) {
    const uint4* g = reinterpret_cast<const uint4*>(p.gate_w + size_t(e) * H);
    float acc[kDecodeMaxT];
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) acc[t] = 0.f;
    for (int c = lane; c < nv; c += 32) {
      float gf[8];
      unpack8(g[c], gf);
#pragma unroll
      for (int t = 0; t < kDecodeMaxT; ++t) {
        if (t < T) {
          const float4* x4 = reinterpret_cast<const float4*>(xn + t * H + c * 8);
          const float4 a = x4[0], b = x4[1];
          acc[t] += gf[0] * a.x + gf[1] * a.y + gf[2] * a.z + gf[3] * a.w + gf[4] * b.x +
                    gf[5] * b.y + gf[6] * b.z + gf[7] * b.w;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) {
      if (t < T) {
        const float v = warp_sum(acc[t]);
        if (lane == 0) p.ws.logits[t * p.E + e] = v;
      }
    }
  }

  // ---- the last router block to finish routes every token
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) am_last = atomicAdd(p.ws.counter, 1u) == unsigned(p.gate_blocks - 1);
  __syncthreads();
  if (!am_last) return;
  __threadfence();
  if (threadIdx.x < T) {
    const int t = threadIdx.x;
    TopK tk;
    tk.init();
    for (int e = 0; e < p.E; ++e)
      tk.offer(e, __ldcg(p.ws.logits + t * p.E + e), p.gate_bias ? p.gate_bias[e] : 0.f, p.k);
    tk.write(p.k, p.rsf, p.ws.idx + t * p.k, p.ws.w + t * p.k);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.umax * kDecodeMaxT; ++i) p.ws.slot_pair[i] = -1;
    int n = 0;
    for (int t = 0; t < T; ++t) {
      for (int j = 0; j < p.k; ++j) {
        const int e = p.ws.idx[t * p.k + j];
        int s = 0;
        while (s < n && p.ws.slot_expert[s] != e) ++s;
        if (s == n) p.ws.slot_expert[n++] = e;
        p.ws.slot_pair[s * kDecodeMaxT + t] = t * p.k + j;
      }
    }
    *p.ws.n_slots = n;
    *p.ws.counter = 0u;
  }
}

struct UpParams {
  const bf16* up_w;    // [E, I, H]
  DecodeWorkspace ws;
  int H, I, k;
};

// grid (ceil(I / 32), umax)
__global__ void __launch_bounds__(kThreads) decode_up(const UpParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ const bf16* src[kDecodeMaxT];
  __shared__ bf16* dst[kDecodeMaxT];
  __shared__ int cnt;
  const int slot = blockIdx.y;
  if (slot >= *p.ws.n_slots) return;
  const int e = p.ws.slot_expert[slot];
  if (threadIdx.x == 0) {
    int n = 0;
    for (int t = 0; t < kDecodeMaxT; ++t) {
      const int pr = p.ws.slot_pair[slot * kDecodeMaxT + t];
      if (pr >= 0) {
        src[n] = p.ws.normed + size_t(t) * p.H;
        dst[n] = p.ws.uo + size_t(pr) * p.I;
        ++n;
      }
    }
    cnt = n;
  }
  __syncthreads();
  bf16* xs = reinterpret_cast<bf16*>(dsm);
  stage_rows(xs, src, cnt, p.H);
  __syncthreads();
  const bf16* W = p.up_w + size_t(e) * p.I * p.H;
  MOE_DISPATCH_NT(cnt, (up_rows<NT>(W, p.H, p.I, blockIdx.x * kRowsPerBlock, xs, dst)));
}

struct DownParams {
  const bf16* down_w;         // [E, H, I]
  const bf16* shared_down_w;  // [H, S]
  DecodeWorkspace ws;
  int T, H, I, S, umax;
};

// grid (ceil(H / 32), umax + 1); slot umax is the shared expert.
__global__ void __launch_bounds__(kThreads) decode_down(const DownParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ const bf16* src[kDecodeMaxT];
  __shared__ float* dst[kDecodeMaxT];
  __shared__ int cnt;
  const int slot = blockIdx.y;
  const bool shared = slot == p.umax;
  if (!shared && slot >= *p.ws.n_slots) return;
  if (threadIdx.x == 0) {
    int n = 0;
    if (shared) {
      for (int t = 0; t < p.T; ++t) {
        src[n] = p.ws.vo + size_t(t) * p.S;
        dst[n] = p.ws.sh + size_t(t) * p.H;
        ++n;
      }
    } else {
      for (int t = 0; t < kDecodeMaxT; ++t) {
        const int pr = p.ws.slot_pair[slot * kDecodeMaxT + t];
        if (pr >= 0) {
          src[n] = p.ws.uo + size_t(pr) * p.I;
          dst[n] = p.ws.ypart + size_t(pr) * p.H;
          ++n;
        }
      }
    }
    cnt = n;
  }
  __syncthreads();
  const int K = shared ? p.S : p.I;
  bf16* xs = reinterpret_cast<bf16*>(dsm);
  stage_rows(xs, src, cnt, K);
  __syncthreads();
  const bf16* W =
      shared ? p.shared_down_w : p.down_w + size_t(p.ws.slot_expert[slot]) * p.H * p.I;
  MOE_DISPATCH_NT(cnt, (down_rows<NT>(W, K, p.H, blockIdx.x * kRowsPerBlock, xs, dst)));
}

// hidden[t] = bf16(residual[t] + sh[t] + sum_j w[t,j] * ypart[t*k + j])
__global__ void decode_combine(const DecodeWorkspace ws, const bf16* residual, bf16* hidden,
                               int T, int H, int k) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;  // element index in [0, T*H)
  if (i >= T * H) return;
  const int t = i / H, h = i - t * H;
  float acc = __bfloat162float(residual[i]) + ws.sh[size_t(t) * H + h];
  for (int j = 0; j < k; ++j)
    acc += ws.w[t * k + j] * ws.ypart[size_t(t * k + j) * H + h];
  hidden[i] = __float2bfloat16_rn(acc);
}

size_t route_smem(int T, int H) {
  const size_t a = size_t(T) * H * 4, b = size_t(T) * H * 2;
  return a > b ? a : b;
}

constexpr size_t kMaxDecodeSmem = 200 * 1024;

}  // namespace

bool decode_supported(const moe_config& c) {
  if (c.latent_size != 0 || c.expert_wdtype != MOE_WEIGHTS_BF16) return false;
  const size_t H = c.hidden_size, I = c.moe_inter, S = c.shared_inter;
  return route_smem(kDecodeMaxT, c.hidden_size) <= kMaxDecodeSmem &&
         kDecodeMaxT * H * 2 <= kMaxDecodeSmem && kDecodeMaxT * I * 2 <= kMaxDecodeSmem &&
         kDecodeMaxT * S * 2 <= kMaxDecodeSmem;
}

cudaError_t prepare_decode() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(decode_route_shared_up, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kMaxDecodeSmem))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(decode_up, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kMaxDecodeSmem))) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(decode_down, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(kMaxDecodeSmem));
}

moe_status enqueue_decode(const DecodeArgs& a, bf16* hidden, bf16* residual, int T,
                          cudaStream_t stream, int* launches) {
  const moe_config& c = *a.cfg;
  if (!decode_supported(c) || T < 1 || T > kDecodeMaxT) return MOE_ERR_INVALID_CONFIG;
  const int H = c.hidden_size, E = c.num_experts, k = c.top_k, I = c.moe_inter,
            S = c.shared_inter;
  const int umax = T * k < E ? T * k : E;

  RouteParams rp;
  rp.hidden = hidden;
  rp.norm_w = static_cast<const bf16*>(a.w->norm_w);
  rp.gate_w = static_cast<const bf16*>(a.w->gate_w);
  rp.gate_bias = a.w->gate_bias;
  rp.shared_up_w = static_cast<const bf16*>(a.w->shared_up_w);
  rp.residual = residual;
  rp.ws = *a.ws;
  rp.T = T;
  rp.H = H;
  rp.E = E;
  rp.k = k;
  rp.S = S;
  rp.umax = umax;
  rp.gate_blocks = (E + kWarps - 1) / kWarps;
  rp.eps = c.rms_eps;
  rp.rsf = c.routed_scaling_factor;
  const int shared_blocks = (S + kRowsPerBlock - 1) / kRowsPerBlock;
  decode_route_shared_up<<<rp.gate_blocks + shared_blocks, kThreads, route_smem(T, H), stream>>>(
      rp);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

  UpParams up;
  up.up_w = static_cast<const bf16*>(a.w->up_w);
  up.ws = *a.ws;
  up.H = H;
  up.I = I;
  up.k = k;
  decode_up<<<dim3((I + kRowsPerBlock - 1) / kRowsPerBlock, umax), kThreads,
              size_t(T) * H * 2, stream>>>(up);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

  DownParams dp;
  dp.down_w = static_cast<const bf16*>(a.w->down_w);
  dp.shared_down_w = static_cast<const bf16*>(a.w->shared_down_w);
  dp.ws = *a.ws;
  dp.T = T;
  dp.H = H;
  dp.I = I;
  dp.S = S;
  dp.umax = umax;
  const size_t dsm = size_t(T) * (I > S ? I : S) * 2;
  decode_down<<<dim3((H + kRowsPerBlock - 1) / kRowsPerBlock, umax + 1), kThreads, dsm,
                stream>>>(dp);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

  decode_combine<<<(T * H + 255) / 256, 256, 0, stream>>>(*a.ws, residual, hidden, T, H, k);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  *launches += 4;
  return MOE_OK;
}

}  // namespace moe
