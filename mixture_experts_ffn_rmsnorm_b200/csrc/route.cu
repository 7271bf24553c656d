// Bandwidth-bound kernels of the prefill path: RMSNorm (with the split
// router input), the stable sort by expert, the row gather feeding the
// grouped up-GEMM, and the unpermute + weighted reduce fused with the shared
// expert and the residual add.
#include <cuda_fp8.h>

#include "../../include/moe_b200.h"
#include "moe_internal.h"
#include "ptx.cuh"
#include "topk.cuh"

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

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  __syncthreads();  // red may still be read by the previous reduction
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    float x = threadIdx.x < kNormThreads / 32 ? red[threadIdx.x] : 0.f;  // identity of both
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float w = __shfl_xor_sync(0xffffffffu, x, o);
      x = is_max ? fmaxf(x, w) : x + w;
    }
    if (threadIdx.x == 0) red[0] = x;
  }
  __syncthreads();
  return red[0];
}

// E4M3 bits of x (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xFFFFu) | (hi << 16);
}

// RMSNorm of one token per block (NemotronMoeLayer `prefill`: rms_norm_residual
// writes the normed activations and the residual).  residual <- hidden; the
// factor r = rsqrt(mean(x^2) + eps) goes to rs[t], and the normed vector
// n = x * r * w, rounded to BF16, to the first H columns of gate_a [T, 2H]
// (the experts', the shared expert's and fc1's input).  The router does not
// read n: it multiplies the raw x by the gate with w folded in and applies r
// to its logits (prep_gate_kernel).  With FP8 experts it also writes an E4M3
// copy of n with one float scale per token (scale = max|n| / 448).
// hist_clear[0..n_clear) is zeroed.  The next launch (the router, whose main
// loop reads only x and the gate) may start at once.
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(
    const __nv_bfloat16* __restrict__ hidden, const __nv_bfloat16* __restrict__ norm_w,
    __nv_bfloat16* __restrict__ residual, __nv_bfloat16* __restrict__ gate_a,
    float* __restrict__ rs, uint8_t* __restrict__ normed_q, float* __restrict__ normed_scale,
    int H, float eps, int* __restrict__ hist_clear, int n_clear) {
  pdl_trigger();
  __shared__ float red[kNormThreads / 32];
  const int t = blockIdx.x;
  for (int i = t * kNormThreads + threadIdx.x; i < n_clear; i += gridDim.x * kNormThreads)
    hist_clear[i] = 0;
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
  const float r = rsqrtf(block_reduce(ss, red, false) / float(H) + eps);
  if (threadIdx.x == 0) rs[t] = r;
  const uint4* w = reinterpret_cast<const uint4*>(norm_w);
  uint4* hi = reinterpret_cast<uint4*>(gate_a + size_t(t) * 2 * H);
  float amax = 0.f;
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    float f[8], g[8], h[8];
    unpack8(x[i], f);
    unpack8(w[i], g);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      h[j] = f[j] * r * g[j];
      amax = fmaxf(amax, fabsf(h[j]));
    }
    hi[i] = pack8(h);
  }
  if (!normed_q) return;
  amax = block_reduce(amax, red, true);
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  const float inv = 1.f / scale;
  if (threadIdx.x == 0) normed_scale[t] = scale;
  uint2* q = reinterpret_cast<uint2*>(normed_q + size_t(t) * H);
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    float f[8], g[8], n[8];
    unpack8(x[i], f);
    unpack8(w[i], g);
#pragma unroll
    for (int j = 0; j < 8; ++j) n[j] = f[j] * r * g[j] * inv;
    q[i] = make_uint2(e4m3x4(n[0], n[1], n[2], n[3]), e4m3x4(n[4], n[5], n[6], n[7]));
  }
}

// The same RMSNorm with the token's chunks of x and of the norm weight held
// in registers (H <= kNormThreads * 8 * MAXC): x is read from memory once and
// the weight load overlaps it, ahead of the block reduction.  Identical
// arithmetic and summation order, hence identical results.
template <int MAXC>
__global__ void __launch_bounds__(kNormThreads) rmsnorm_reg_kernel(
    const __nv_bfloat16* __restrict__ hidden, const __nv_bfloat16* __restrict__ norm_w,
    __nv_bfloat16* __restrict__ residual, __nv_bfloat16* __restrict__ gate_a,
    float* __restrict__ rs, uint8_t* __restrict__ normed_q, float* __restrict__ normed_scale,
    int H, float eps, int* __restrict__ hist_clear, int n_clear) {
  pdl_trigger();
  __shared__ float red[kNormThreads / 32];
  const int t = blockIdx.x;
  for (int i = t * kNormThreads + threadIdx.x; i < n_clear; i += gridDim.x * kNormThreads)
    hist_clear[i] = 0;
  const uint4* x = reinterpret_cast<const uint4*>(hidden + size_t(t) * H);
  const uint4* w = reinterpret_cast<const uint4*>(norm_w);
  uint4* res = reinterpret_cast<uint4*>(residual + size_t(t) * H);
  const int nv = H / 8;
  uint4 xv[MAXC], wv[MAXC];
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int i = threadIdx.x + c * kNormThreads;
    if (i < nv) {
      xv[c] = x[i];
      wv[c] = w[i];
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int i = threadIdx.x + c * kNormThreads;
    if (i < nv) {
      res[i] = xv[c];
      float f[8];
      unpack8(xv[c], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss += f[j] * f[j];
    }
  }
  const float r = rsqrtf(block_reduce(ss, red, false) / float(H) + eps);
  if (threadIdx.x == 0) rs[t] = r;
  uint4* hi = reinterpret_cast<uint4*>(gate_a + size_t(t) * 2 * H);
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int i = threadIdx.x + c * kNormThreads;
    if (i < nv) {
      float f[8], g[8], h[8];
      unpack8(xv[c], f);
      unpack8(wv[c], g);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        h[j] = f[j] * r * g[j];
        amax = fmaxf(amax, fabsf(h[j]));
      }
      hi[i] = pack8(h);
    }
  }
  if (!normed_q) return;
  amax = block_reduce(amax, red, true);
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  const float inv = 1.f / scale;
  if (threadIdx.x == 0) normed_scale[t] = scale;
  uint2* q = reinterpret_cast<uint2*>(normed_q + size_t(t) * H);
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int i = threadIdx.x + c * kNormThreads;
    if (i < nv) {
      float f[8], g[8], n[8];
      unpack8(xv[c], f);
      unpack8(wv[c], g);
#pragma unroll
      for (int j = 0; j < 8; ++j) n[j] = f[j] * r * g[j] * inv;
      q[i] = make_uint2(e4m3x4(n[0], n[1], n[2], n[3]), e4m3x4(n[4], n[5], n[6], n[7]));
    }
  }
}

// The router's gate with the norm weight folded in, as two BF16 halves
// (once, when the layer is created): g'[e, i] = G[e, i] * w[i] in fp32,
// out[e] = [bf16(g') | bf16(g' - bf16(g'))] [E, 2H].  The router multiplies
// the token rows x (BF16, exact) by both halves, so that it sums
// x_i * g'_ei to about 16 significant bits per term: with r applied to the
// sum, logit = r * (G . (x * w)) = G . n in float32 accuracy.
__global__ void prep_gate_kernel(const __nv_bfloat16* __restrict__ gate,
                                 const __nv_bfloat16* __restrict__ norm_w, int E, int H,
                                 __nv_bfloat16* __restrict__ out) {
  const size_t n = size_t(E) * H;
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x) {
    const size_t e = i / H, c = i - e * H;
    const float g = __bfloat162float(gate[i]) * __bfloat162float(norm_w[c]);
    const __nv_bfloat16 hi = __float2bfloat16_rn(g);
    out[e * 2 * H + c] = hi;
    out[e * 2 * H + H + c] = __float2bfloat16_rn(g - __bfloat162float(hi));
  }
}

// Split-K router, second half (one warp per token).  Lane l sums the
// partial logits of experts l, l + 32, ... over the splits in split order
// (two splits' loads in flight at a time, each warp load one coalesced
// 128-byte row segment), then the warp runs the sigmoid top-k on the sums
// and adds the token's choices to its 128-token tile's expert histogram.
__global__ void __launch_bounds__(256) router_reduce_kernel(
    const float* __restrict__ part, int ks, int rows_cap, int T, int E,
    const float* __restrict__ bias, int k, float rsf, const float* __restrict__ rs,
    int* __restrict__ idx, float* __restrict__ w, int* __restrict__ hist) {
  pdl_wait();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  const size_t sstride = size_t(rows_cap) * E;
  const float* src = part + size_t(t) * E + lane;
  const int nj = (E + 31) / 32;  // experts per lane (<= 8)
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  // splits in order, two at a time so that their loads are in flight together
  int s = 0;
  for (; s + 2 <= ks; s += 2) {
    float a[8], b[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      a[j] = j < nj && lane + 32 * j < E ? __ldcg(src + size_t(s) * sstride + 32 * j) : 0.f;
      b[j] = j < nj && lane + 32 * j < E ? __ldcg(src + size_t(s + 1) * sstride + 32 * j) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = (acc[j] + a[j]) + b[j];
  }
  if (s < ks) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      acc[j] += j < nj && lane + 32 * j < E ? __ldcg(src + size_t(s) * sstride + 32 * j) : 0.f;
  }
  // the partials are G' . x: the token's factor r makes them the logits
  const float r = rs[t];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] *= r;
  const int e = warp_topk_regs(acc, bias, E, k, rsf, idx + size_t(t) * k, w + size_t(t) * k);
  // (an out-of-range id comes only from NaN logits; the sort flags it)
  if (lane < k && unsigned(e) < unsigned(E)) atomicAdd(hist + size_t(t / kBM) * E + e, 1);
}

// E4M3 copy of a row set: q[p] = E4M3(x[p] / s_p), s_p = amax_p / 448, and
// amax_p reset to 0 for the next forward.  One warp per row, eight rows per
// block, each lane with up to kBatch 8-element chunks in flight; rows
// [0, R) are those of the first set (routed relu^2(up), width I), rows
// [R, R + Rv) those of the second (shared relu^2(up), width S).  (A block
// per row left most threads with one or two chunks: 62 us for the skewed
// FP8 workload's 49152 rows of 1856.)
constexpr int kQuantRows = 8;  // rows (warps) per block of quantize_rows_kernel

__global__ void quantize_rows_kernel(const __nv_bfloat16* __restrict__ u,
                                     unsigned* __restrict__ u_amax, uint8_t* __restrict__ uq,
                                     float* __restrict__ u_scale, int R, int I,
                                     const __nv_bfloat16* __restrict__ v,
                                     unsigned* __restrict__ v_amax, uint8_t* __restrict__ vq,
                                     float* __restrict__ v_scale, int Rv, int S) {
  const int lane = threadIdx.x & 31;
  int p = blockIdx.x * kQuantRows + (threadIdx.x >> 5);
  if (p >= R + Rv) return;  // (no block-wide barrier below)
  const __nv_bfloat16* x = u;
  unsigned* amax = u_amax;
  uint8_t* q = uq;
  float* scale = u_scale;
  int W = I;
  if (p >= R) {
    p -= R;
    x = v;
    amax = v_amax;
    q = vq;
    scale = v_scale;
    W = S;
  }
  const float m = __uint_as_float(amax[p]);
  const float s = m > 0.f ? m / 448.f : 1.f;
  const float inv = 1.f / s;
  const uint4* src = reinterpret_cast<const uint4*>(x + size_t(p) * W);
  uint2* dst = reinterpret_cast<uint2*>(q + size_t(p) * W);
  // kBatch chunks of 8 per lane in flight before the first conversion
  constexpr int kBatch = 8;
  const int nv = W / 8;
  for (int i0 = lane; i0 < nv; i0 += kBatch * 32) {
    uint4 xv[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int i = i0 + b * 32;
      if (i < nv) xv[b] = __ldcs(src + i);
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int i = i0 + b * 32;
      if (i < nv) {
        float f[8];
        unpack8(xv[b], f);
        dst[i] = make_uint2(e4m3x4(f[0] * inv, f[1] * inv, f[2] * inv, f[3] * inv),
                            e4m3x4(f[4] * inv, f[5] * inv, f[6] * inv, f[7] * inv));
      }
    }
  }
  __syncwarp();  // (every lane has read amax[p])
  if (lane == 0) {
    scale[p] = s;
    amax[p] = 0u;
  }
}

constexpr int kSortThreads = 512;
constexpr int kSortWarps = kSortThreads / 32;

// Expert histogram of each 128-token tile of a routing table (the router
// GEMM's epilogue produces the same table during a forward pass).
__global__ void tile_hist_kernel(const int* __restrict__ idx, int T, int k, int E,
                                 int* __restrict__ hist, int* __restrict__ status) {
  __shared__ int h[MOE_MAX_EXPERTS];
  const int mt = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int f0 = mt * kBM * k, f1 = min(T, (mt + 1) * kBM) * k;
  for (int f = f0 + threadIdx.x; f < f1; f += blockDim.x) {
    const int e = idx[f];
    if (unsigned(e) < unsigned(E))
      atomicAdd(&h[e], 1);
    else
      atomicOr(status, kStatusBadIndex);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[size_t(mt) * E + e] = h[e];
}

// Stable sort of the R = T*k routed rows by expert, one CTA per 128-token
// tile.  From the per-tile expert histograms every CTA derives the global
// per-expert offsets (exclusive prefix over experts) and its own base
// (prefix over earlier tiles); inside its tile, warps take contiguous row
// segments with per-warp histograms and scatter 32 rows at a time, ranking
// equal experts with __match_any_sync, so rows keep token order inside every
// expert.  CTA 0 also writes off[E + 1] and the grouped GEMM's m-tile table
// (ceil(count_e / 128) tiles per expert, in expert order).
__global__ void __launch_bounds__(kSortThreads) sort_tiles_kernel(
    const int* __restrict__ idx, const int* __restrict__ hist, int T, int k, int E,
    int* __restrict__ perm, int* __restrict__ inv, int* __restrict__ off,
    int2* __restrict__ tile_table, int* __restrict__ n_mtiles, int* __restrict__ status) {
  __shared__ int base[MOE_MAX_EXPERTS];
  __shared__ int tot[MOE_MAX_EXPERTS + 1];
  __shared__ int toff[MOE_MAX_EXPERTS + 1];
  __shared__ int wh[kSortWarps][MOE_MAX_EXPERTS];  // per-warp counts, then cursors
  const int mt = blockIdx.x, ntiles = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < E; e += kSortThreads) {
    int before = 0, all = 0;
    for (int m = 0; m < ntiles; ++m) {
      const int c = hist[size_t(m) * E + e];
      all += c;
      if (m < mt) before += c;
    }
    tot[e] = all;
    base[e] = before;
  }
  for (int i = threadIdx.x; i < kSortWarps * E; i += kSortThreads) wh[i / E][i % E] = 0;
  __syncthreads();
  if (warp == 0) {  // exclusive scans over experts: rows and 128-row tiles
    int acc = 0, tacc = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < E ? tot[e] : 0;
      int inc = c, tinc = (c + kBM - 1) / kBM;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        const int z = __shfl_up_sync(0xffffffffu, tinc, o);
        if (lane >= o) {
          inc += y;
          tinc += z;
        }
      }
      if (e < E) {
        toff[e] = tacc + tinc - (c + kBM - 1) / kBM;
        base[e] += acc + inc - c;
        if (mt == 0) off[e] = acc + inc - c;
      }
      acc += __shfl_sync(0xffffffffu, inc, 31);
      tacc += __shfl_sync(0xffffffffu, tinc, 31);
    }
    if (lane == 0) {
      toff[E] = tacc;
      if (mt == 0) {
        off[E] = acc;
        *n_mtiles = tacc;
      }
    }
  }
  __syncthreads();
  if (mt == 0) {
    for (int e = threadIdx.x; e < E; e += kSortThreads) {
      const int o = base[e];  // tile 0: its base is the global offset
      for (int i = toff[e]; i < toff[e + 1]; ++i) tile_table[i] = make_int2(e, o + (i - toff[e]) * kBM);
    }
  }
  // this tile's rows, in row order
  const int f0 = mt * kBM * k, f1 = min(T, (mt + 1) * kBM) * k;
  const int seg = (f1 - f0 + kSortWarps - 1) / kSortWarps;
  const int g0 = min(f1, f0 + warp * seg), g1 = min(f1, g0 + seg);
  for (int f = g0 + lane; f < g1; f += 32) {
    const int e = idx[f];
    if (unsigned(e) < unsigned(E)) atomicAdd(&wh[warp][e], 1);
    else atomicOr(status, kStatusBadIndex);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kSortThreads) {
    int b = base[e];
    for (int w = 0; w < kSortWarps; ++w) {
      const int c = wh[w][e];
      wh[w][e] = b;
      b += c;
    }
  }
  __syncthreads();
  for (int g = g0; g < g1; g += 32) {
    const int f = g + lane;
    int e = f < g1 ? idx[f] : -1;
    if (unsigned(e) >= unsigned(E)) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0) {
      const int pos = wh[warp][e] + rank;
      if (pos >= 0 && pos < T * k) {
        perm[pos] = f;
        inv[f] = pos;
      } else {
        inv[f] = -1;
        atomicOr(status, kStatusBadIndex);  // inconsistent histogram: skip the write
      }
    } else if (f < g1) {
      inv[f] = -1;  // an id outside [0, E) (only from NaN logits): the row goes nowhere
    }
    __syncwarp();
    if (e >= 0 && rank == 0) wh[warp][e] += __popc(peers);
    __syncwarp();
  }
}

// xs[p, :] = X[perm[p] / k, :] (row_bytes per row): one warp per sorted
// row, 16-byte moves; with FP8 inputs the token scale travels along.
__global__ void gather_kernel(const uint8_t* __restrict__ X, size_t ldx,
                              const int* __restrict__ perm, int k, int R, int row_bytes,
                              uint8_t* __restrict__ xs, const float* __restrict__ scale,
                              float* __restrict__ xs_scale) {
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (p >= R) return;
  const int lane = threadIdx.x & 31;
  const int t = perm[p] / k;
  const uint4* src = reinterpret_cast<const uint4*>(X + size_t(t) * ldx);
  uint4* dst = reinterpret_cast<uint4*>(xs + size_t(p) * row_bytes);
  // kBatch loads per lane in flight before the first store
  constexpr int kBatch = 4;
  const int nv = row_bytes / 16;
  for (int i0 = lane; i0 < nv; i0 += kBatch * 32) {
    uint4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (i0 + b * 32 < nv) v[b] = src[i0 + b * 32];
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
      if (i0 + b * 32 < nv) dst[i0 + b * 32] = v[b];
  }
  if (scale && lane == 0) xs_scale[p] = scale[t];
}

// Token t's slot j (thread j < k): its sorted row and weight into rows /
// wts.  A slot whose expert id was out of range (only from non-finite
// logits; the sort then sets its inv to -1 and reports it) reads row 0,
// inside the buffer, with weight 0 (it adds 0 unless that row holds a
// non-finite value, which only the outputs of such a token may then show).
// The loop over the slots stays branch-free.
__device__ __forceinline__ void load_slot(const int* __restrict__ inv, const float* __restrict__ w,
                                          int t, int k, int R, int* rows, float* wts) {
  const int j = threadIdx.x;
  if (j < k) {
    const int r = inv[t * k + j];
    const float wv = w[t * k + j];  // (both loads in flight at once)
    const bool ok = r >= 0 && r < R;
    rows[j] = ok ? r : 0;
    wts[j] = ok ? wv : 0.f;
  }
}

// hidden[t] = bf16(residual[t] + s[t] + sum_j w[t,j] * y[inv[t*k + j]])
// (MoeLayer `forward_prefill`: unpermute + weighted reduce, shared expert
// blend; nemotron_moe.rs module documentation: summed and added to hidden).
__global__ void combine_kernel(const __nv_bfloat16* __restrict__ y, const int* __restrict__ inv,
                               const float* __restrict__ w, const float* __restrict__ s,
                               const __nv_bfloat16* __restrict__ residual,
                               __nv_bfloat16* __restrict__ hidden, int k, int H, int R) {
  const int t = blockIdx.x;
  __shared__ int rows[kMaxTopKShared];
  __shared__ float wts[kMaxTopKShared];
  load_slot(inv, w, t, k, R, rows, wts);
  __syncthreads();
  const int nv = H / 8;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    float acc[8], f[8];
    unpack8(reinterpret_cast<const uint4*>(residual + size_t(t) * H)[i], acc);
    const float4* s4 = reinterpret_cast<const float4*>(s + size_t(t) * H) + 2 * i;
    const float4 a = s4[0], b = s4[1];
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    // two rows' loads in flight per step (the same order of additions)
    int j = 0;
    for (; j + 2 <= k; j += 2) {
      const uint4 ya = __ldcs(reinterpret_cast<const uint4*>(y + size_t(rows[j]) * H) + i);
      const uint4 yb = __ldcs(reinterpret_cast<const uint4*>(y + size_t(rows[j + 1]) * H) + i);
      float fb[8];
      unpack8(ya, f);
      unpack8(yb, fb);
      const float wa = wts[j], wb = wts[j + 1];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wa * f[q];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wb * fb[q];
    }
    if (j < k) {
      unpack8(__ldcs(reinterpret_cast<const uint4*>(y + size_t(rows[j]) * H) + i), f);
      const float wj = wts[j];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wj * f[q];
    }
    reinterpret_cast<uint4*>(hidden + size_t(t) * H)[i] = pack8(acc);
  }
}

// LatentMoE: m[t] = bf16(sum_j w[t,j] * y[inv[t*k + j]]) in latent space.
// With FP8 fc2 weights the block also writes the row's E4M3 copy mq[t] with
// its scale (max |m[t]| / 448): the block owns the whole row.
__global__ void latent_reduce_kernel(const __nv_bfloat16* __restrict__ y,
                                     const int* __restrict__ inv, const float* __restrict__ w,
                                     __nv_bfloat16* __restrict__ m, uint8_t* __restrict__ mq,
                                     float* __restrict__ m_scale, int k, int L, int R) {
  const int t = blockIdx.x;
  __shared__ int rows[kMaxTopKShared];
  __shared__ float wts[kMaxTopKShared];
  __shared__ float red[32];
  load_slot(inv, w, t, k, R, rows, wts);
  __syncthreads();
  const int nv = L / 8;
  float amax = 0.f;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, f[8];
    // two rows' loads in flight per step (the same order of additions)
    int j = 0;
    for (; j + 2 <= k; j += 2) {
      const uint4 ya = __ldcs(reinterpret_cast<const uint4*>(y + size_t(rows[j]) * L) + i);
      const uint4 yb = __ldcs(reinterpret_cast<const uint4*>(y + size_t(rows[j + 1]) * L) + i);
      float fb[8];
      unpack8(ya, f);
      unpack8(yb, fb);
      const float wa = wts[j], wb = wts[j + 1];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wa * f[q];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wb * fb[q];
    }
    if (j < k) {
      unpack8(__ldcs(reinterpret_cast<const uint4*>(y + size_t(rows[j]) * L) + i), f);
      const float wj = wts[j];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += wj * f[q];
    }
    const uint4 packed = pack8(acc);
    reinterpret_cast<uint4*>(m + size_t(t) * L)[i] = packed;
    unpack8(packed, f);
#pragma unroll
    for (int q = 0; q < 8; ++q) amax = fmaxf(amax, fabsf(f[q]));
  }
  if (!mq) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  float a = 0.f;
  for (int i = 0; i < int(blockDim.x >> 5); ++i) a = fmaxf(a, red[i]);
  const float scale = a > 0.f ? a / 448.f : 1.f;
  const float rcp = 1.f / scale;
  if (threadIdx.x == 0) m_scale[t] = scale;
  // the E4M3 copy of the bf16 row this thread wrote above
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    float f[8];
    unpack8(reinterpret_cast<const uint4*>(m + size_t(t) * L)[i], f);
    reinterpret_cast<uint2*>(mq + size_t(t) * L)[i] =
        make_uint2(e4m3x4(f[0] * rcp, f[1] * rcp, f[2] * rcp, f[3] * rcp),
                   e4m3x4(f[4] * rcp, f[5] * rcp, f[6] * rcp, f[7] * rcp));
  }
}

}  // namespace

cudaError_t launch_rmsnorm(const __nv_bfloat16* hidden, const __nv_bfloat16* norm_w,
                           __nv_bfloat16* residual, __nv_bfloat16* gate_a, float* rs,
                           uint8_t* normed_q, float* normed_scale, int T, int H, float eps,
                           int* hist_clear, int n_clear, cudaStream_t stream) {
  const int nc = hist_clear ? n_clear : 0;
  const int chunks = (H / 8 + kNormThreads - 1) / kNormThreads;
  if (chunks <= 2)
    rmsnorm_reg_kernel<2><<<T, kNormThreads, 0, stream>>>(hidden, norm_w, residual, gate_a, rs,
                                                          normed_q, normed_scale, H, eps,
                                                          hist_clear, nc);
  else if (chunks <= 8)
    rmsnorm_reg_kernel<8><<<T, kNormThreads, 0, stream>>>(hidden, norm_w, residual, gate_a, rs,
                                                          normed_q, normed_scale, H, eps,
                                                          hist_clear, nc);
  else
    rmsnorm_kernel<<<T, kNormThreads, 0, stream>>>(hidden, norm_w, residual, gate_a, rs,
                                                   normed_q, normed_scale, H, eps, hist_clear,
                                                   nc);
  return cudaGetLastError();
}

cudaError_t launch_prep_gate(const __nv_bfloat16* gate, const __nv_bfloat16* norm_w, int E, int H,
                             __nv_bfloat16* out, cudaStream_t stream) {
  prep_gate_kernel<<<592, 256, 0, stream>>>(gate, norm_w, E, H, out);
  return cudaGetLastError();
}

cudaError_t launch_router_reduce(const float* part, int ks, int rows_cap, int T, int E,
                                 const float* bias, int k, float rsf, const float* rs, int* idx,
                                 float* w, int* hist, cudaStream_t stream) {
  if (ks < 2 || ks > kRouterMaxSplit || E > 256) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((T + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_reduce_kernel, part, ks, rows_cap, T, E, bias, k, rsf,
                            rs, idx, w, hist);
}

cudaError_t launch_quantize_rows(const __nv_bfloat16* u, unsigned* u_amax, uint8_t* uq,
                                 float* u_scale, int R, int I, const __nv_bfloat16* v,
                                 unsigned* v_amax, uint8_t* vq, float* v_scale, int Rv, int S,
                                 cudaStream_t stream) {
  if (R + Rv <= 0) return cudaSuccess;
  quantize_rows_kernel<<<(R + Rv + kQuantRows - 1) / kQuantRows, 32 * kQuantRows, 0, stream>>>(
      u, u_amax, uq, u_scale, R, I, v, v_amax, vq, v_scale, Rv, S);
  return cudaGetLastError();
}

cudaError_t launch_tile_hist(const int* idx, int T, int k, int E, int* hist, int* status,
                             cudaStream_t stream) {
  tile_hist_kernel<<<(T + kBM - 1) / kBM, 256, 0, stream>>>(idx, T, k, E, hist, status);
  return cudaGetLastError();
}

cudaError_t launch_sort(const int* idx, const int* hist, int T, int k, int E, int* perm, int* inv,
                        int* off, int2* tile_table, int* n_mtiles, int* status,
                        cudaStream_t stream) {
  sort_tiles_kernel<<<(T + kBM - 1) / kBM, kSortThreads, 0, stream>>>(
      idx, hist, T, k, E, perm, inv, off, tile_table, n_mtiles, status);
  return cudaGetLastError();
}

cudaError_t launch_gather(const void* X, size_t ldx_bytes, const int* perm, int k, int R,
                          int row_bytes, void* xs, const float* scale, float* xs_scale,
                          cudaStream_t stream) {
  const int warps = 8;
  gather_kernel<<<(R + warps - 1) / warps, warps * 32, 0, stream>>>(
      static_cast<const uint8_t*>(X), ldx_bytes, perm, k, R, row_bytes,
      static_cast<uint8_t*>(xs), scale, xs_scale);
  return cudaGetLastError();
}

cudaError_t launch_combine(const __nv_bfloat16* y, const int* inv, const float* w, const float* s,
                           const __nv_bfloat16* residual, __nv_bfloat16* hidden, int T, int k,
                           int H, cudaStream_t stream) {
  combine_kernel<<<T, 128, 0, stream>>>(y, inv, w, s, residual, hidden, k, H, T * k);
  return cudaGetLastError();
}

cudaError_t launch_latent_reduce(const __nv_bfloat16* y, const int* inv, const float* w,
                                 __nv_bfloat16* m, uint8_t* mq, float* m_scale, int T, int k,
                                 int L, cudaStream_t stream) {
  latent_reduce_kernel<<<T, 128, 0, stream>>>(y, inv, w, m, mq, m_scale, k, L, T * k);
  return cudaGetLastError();
}

}  // namespace moe
