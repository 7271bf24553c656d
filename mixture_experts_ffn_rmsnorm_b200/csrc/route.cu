// Bandwidth-bound kernels of the prefill path: RMSNorm (with the split
// router input), the stable sort by expert, the row gather feeding the
// grouped up-GEMM, and the unpermute + weighted reduce fused with the shared
// expert and the residual add.
#include "moe_internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  f[0] = bf16lo(u.x); f[1] = bf16hi(u.x);
  f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
  f[4] = bf16lo(u.z); f[5] = bf16hi(u.z);
  f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

constexpr int kNormThreads = 256;

// RMSNorm of one token per block (NemotronMoeLayer `prefill`: rms_norm_residual
// writes the normed activations and the residual).  residual <- hidden; the
// normed vector n = x * rsqrt(mean(x^2) + eps) * w is written as two BF16
// halves into gate_a [T, 2H]: hi = bf16(n) (this is also the experts' input)
// and lo = bf16(n - hi), so the router GEMM on [hi | lo] x [G | G] sees n to
// about 16 significant bits (FP32-accurate logits from BF16 tensor cores).
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(
    const __nv_bfloat16* __restrict__ hidden, const __nv_bfloat16* __restrict__ norm_w,
    __nv_bfloat16* __restrict__ residual, __nv_bfloat16* __restrict__ gate_a, int H, float eps) {
  const int t = blockIdx.x;
  const uint4* x = reinterpret_cast<const uint4*>(hidden + size_t(t) * H);
  uint4* res = reinterpret_cast<uint4*>(residual + size_t(t) * H);
  const int nv = H / 8;
  float ss = 0.f;
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    const uint4 u = x[i];
    res[i] = u;
    float f[8];
    unpack8(u, f);
#pragma unroll
    for (int j = 0; j < 8; ++j) ss += f[j] * f[j];
  }
  __shared__ float red[kNormThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < kNormThreads / 32 ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float r = rsqrtf(red[0] / float(H) + eps);
  const uint4* w = reinterpret_cast<const uint4*>(norm_w);
  uint4* hi = reinterpret_cast<uint4*>(gate_a + size_t(t) * 2 * H);
  uint4* lo = hi + nv;
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    float f[8], g[8], h[8], l[8];
    unpack8(x[i], f);
    unpack8(w[i], g);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float n = f[j] * r * g[j];
      h[j] = __bfloat162float(__float2bfloat16_rn(n));
      l[j] = n - h[j];
    }
    hi[i] = pack8(h);
    lo[i] = pack8(l);
  }
}

constexpr int kSortThreads = 1024;
constexpr int kSortWarps = kSortThreads / 32;

// Stable sort of the R = T*k routed rows by expert in one CTA: per-warp
// expert histograms over contiguous row segments, an exclusive prefix over
// (expert, warp), then each warp scatters its segment 32 rows at a time,
// ranking equal experts inside the batch with __match_any_sync so row order
// is kept within every expert.  Also emits the m-tile table of the grouped
// GEMM: ceil(count_e / 128) tiles per expert, in expert order.
__global__ void __launch_bounds__(kSortThreads) sort_kernel(
    const int* __restrict__ idx, int R, int E, int* __restrict__ perm, int* __restrict__ inv,
    int* __restrict__ off, int2* __restrict__ tile_table, int* __restrict__ n_mtiles,
    int* __restrict__ status) {
  extern __shared__ int sm[];
  int* hist = sm;                      // [kSortWarps][E]: counts, then write cursors
  int* eoff = hist + kSortWarps * E;   // [E + 1]
  int* toff = eoff + E + 1;            // [E + 1]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kSortWarps * E; i += kSortThreads) hist[i] = 0;
  __syncthreads();
  const int seg = (R + kSortWarps - 1) / kSortWarps;
  const int f0 = min(R, warp * seg);
  const int f1 = min(R, f0 + seg);
  for (int f = f0 + lane; f < f1; f += 32) {
    const int e = idx[f];
    if (unsigned(e) < unsigned(E))
      atomicAdd(&hist[warp * E + e], 1);
    else
      atomicOr(status, kStatusBadIndex);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kSortThreads) {
    int s = 0;
    for (int w = 0; w < kSortWarps; ++w) s += hist[w * E + e];
    eoff[e] = s;  // count for now
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0, tacc = 0;
    for (int e = 0; e < E; ++e) {
      const int c = eoff[e];
      eoff[e] = acc;
      toff[e] = tacc;
      acc += c;
      tacc += (c + kBM - 1) / kBM;
    }
    eoff[E] = acc;
    toff[E] = tacc;
    *n_mtiles = tacc;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += kSortThreads) off[e] = eoff[e];
  for (int e = threadIdx.x; e < E; e += kSortThreads) {
    int b = eoff[e];
    for (int w = 0; w < kSortWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = b;
      b += c;
    }
    for (int i = toff[e]; i < toff[e + 1]; ++i)
      tile_table[i] = make_int2(e, eoff[e] + (i - toff[e]) * kBM);
  }
  __syncthreads();
  for (int base = f0; base < f1; base += 32) {
    const int f = base + lane;
    const bool valid = f < f1;
    int e = valid ? idx[f] : -1;
    if (unsigned(e) >= unsigned(E)) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0) {
      const int pos = hist[warp * E + e] + rank;
      perm[pos] = f;
      inv[f] = pos;
    }
    __syncwarp();
    if (e >= 0 && rank == 0) hist[warp * E + e] += __popc(peers);
    __syncwarp();
  }
}

// xs[p, :] = X[perm[p] / k, :]: one warp per sorted row, 16-byte moves.
__global__ void gather_kernel(const __nv_bfloat16* __restrict__ X, int ldx,
                              const int* __restrict__ perm, int k, int R, int D,
                              __nv_bfloat16* __restrict__ xs) {
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (p >= R) return;
  const int lane = threadIdx.x & 31;
  const int t = perm[p] / k;
  const uint4* src = reinterpret_cast<const uint4*>(X + size_t(t) * ldx);
  uint4* dst = reinterpret_cast<uint4*>(xs + size_t(p) * D);
  for (int i = lane; i < D / 8; i += 32) dst[i] = src[i];
}

// hidden[t] = bf16(residual[t] + s[t] + sum_j w[t,j] * y[inv[t*k + j]])
// (MoeLayer `forward_prefill`: unpermute + weighted reduce, shared expert
// blend; nemotron_moe.rs module documentation: summed and added to hidden).
__global__ void combine_kernel(const __nv_bfloat16* __restrict__ y, const int* __restrict__ inv,
                               const float* __restrict__ w, const float* __restrict__ s,
                               const __nv_bfloat16* __restrict__ residual,
                               __nv_bfloat16* __restrict__ hidden, int k, int H) {
  const int t = blockIdx.x;
  __shared__ int rows[kMaxTopKShared];
  __shared__ float wts[kMaxTopKShared];
  if (threadIdx.x < k) {
    rows[threadIdx.x] = inv[t * k + threadIdx.x];
    wts[threadIdx.x] = w[t * k + threadIdx.x];
  }
  __syncthreads();
  const int nv = H / 8;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    float acc[8], f[8];
    unpack8(reinterpret_cast<const uint4*>(residual + size_t(t) * H)[i], acc);
    const float4* s4 = reinterpret_cast<const float4*>(s + size_t(t) * H) + 2 * i;
    const float4 a = s4[0], b = s4[1];
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    for (int j = 0; j < k; ++j) {
      unpack8(reinterpret_cast<const uint4*>(y + size_t(rows[j]) * H)[i], f);
      const float wj = wts[j];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wj * f[q];
    }
    reinterpret_cast<uint4*>(hidden + size_t(t) * H)[i] = pack8(acc);
  }
}

// LatentMoE: m[t] = bf16(sum_j w[t,j] * y[inv[t*k + j]]) in latent space.
__global__ void latent_reduce_kernel(const __nv_bfloat16* __restrict__ y,
                                     const int* __restrict__ inv, const float* __restrict__ w,
                                     __nv_bfloat16* __restrict__ m, int k, int L) {
  const int t = blockIdx.x;
  __shared__ int rows[kMaxTopKShared];
  __shared__ float wts[kMaxTopKShared];
  if (threadIdx.x < k) {
    rows[threadIdx.x] = inv[t * k + threadIdx.x];
    wts[threadIdx.x] = w[t * k + threadIdx.x];
  }
  __syncthreads();
  const int nv = L / 8;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, f[8];
    for (int j = 0; j < k; ++j) {
      unpack8(reinterpret_cast<const uint4*>(y + size_t(rows[j]) * L)[i], f);
      const float wj = wts[j];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wj * f[q];
    }
    reinterpret_cast<uint4*>(m + size_t(t) * L)[i] = pack8(acc);
  }
}

}  // namespace

cudaError_t launch_rmsnorm(const __nv_bfloat16* hidden, const __nv_bfloat16* norm_w,
                           __nv_bfloat16* residual, __nv_bfloat16* gate_a, int T, int H,
                           float eps, cudaStream_t stream) {
  rmsnorm_kernel<<<T, kNormThreads, 0, stream>>>(hidden, norm_w, residual, gate_a, H, eps);
  return cudaGetLastError();
}

size_t sort_smem_bytes(int E) { return sizeof(int) * (size_t(kSortWarps) * E + 2 * (E + 1)); }

cudaError_t launch_sort(const int* idx, int T, int k, int E, int* perm, int* inv, int* off,
                        int2* tile_table, int* n_mtiles, int* status, cudaStream_t stream) {
  const size_t smem = sort_smem_bytes(E);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
    if (e != cudaSuccess) return e;
  }
  sort_kernel<<<1, kSortThreads, smem, stream>>>(idx, T * k, E, perm, inv, off, tile_table,
                                                 n_mtiles, status);
  return cudaGetLastError();
}

cudaError_t launch_gather(const __nv_bfloat16* X, int ldx, const int* perm, int k, int R, int D,
                          __nv_bfloat16* xs, cudaStream_t stream) {
  const int warps = 8;
  gather_kernel<<<(R + warps - 1) / warps, warps * 32, 0, stream>>>(X, ldx, perm, k, R, D, xs);
  return cudaGetLastError();
}

cudaError_t launch_combine(const __nv_bfloat16* y, const int* inv, const float* w, const float* s,
                           const __nv_bfloat16* residual, __nv_bfloat16* hidden, int T, int k,
                           int H, cudaStream_t stream) {
  combine_kernel<<<T, 128, 0, stream>>>(y, inv, w, s, residual, hidden, k, H);
  return cudaGetLastError();
}

cudaError_t launch_latent_reduce(const __nv_bfloat16* y, const int* inv, const float* w,
                                 __nv_bfloat16* m, int T, int k, int L, cudaStream_t stream) {
  latent_reduce_kernel<<<T, 128, 0, stream>>>(y, inv, w, m, k, L);
  return cudaGetLastError();
}

}  // namespace moe
