// Decode path, routing kernel (1 <= T <= 8 tokens).
//
// Each warp owns one router row: it issues all of that row's loads first,
// then every block stages x * w_norm (fp32) for the T tokens in shared memory
// while reducing their sums of squares, and the warp computes
// logit = rsqrt(mean x^2 + eps) * (G_e . (x * w)) in fp32, which is the
// logit of the un-rounded normed vector without waiting on the norm.  The last block to
// finish runs a warp-parallel sigmoid top-k per token, groups the routed
// (token, slot) pairs by distinct expert into segments, and writes the
// segment table and the up launch's tile list.  Block 0 writes the
// residual and the bf16 normed rows (the B operand of the up launch).
#include "decode.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxSeg = kDecodeMaxT * kTopKMax + 1;

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

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

struct RouteParams {
  const bf16* hidden;
  const bf16* norm_w;
  const bf16* gate_w;
  const float* gate_bias;
  bf16* residual;
  DecodeWorkspace ws;
  int T, H, E, k, I, S;
  float eps, rsf;
};

constexpr int kRowChunks = 16;  // 16-byte chunks per lane of one router row (H <= 4096)

// MAXT: the token count rounded up to 1, 2, 4 or 8; the per-token loops are
// unrolled to MAXT, which keeps the code of small batches short.
template <int MAXT>
__global__ void __launch_bounds__(kThreads) decode_route(const RouteParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float rs[kDecodeMaxT];
  __shared__ float red[kWarps][kDecodeMaxT];
  __shared__ int am_last;
  __shared__ int s_idx[kMaxSeg];
  __shared__ float s_w[kMaxSeg];
  __shared__ int s_first[kMaxSeg];       // pair f is its expert's first use
  __shared__ int s_seg_of[MOE_MAX_EXPERTS];
  __shared__ int s_exp[kMaxSeg];
  __shared__ int s_nseg;
  __shared__ float s_bias[MOE_MAX_EXPERTS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.H, T = p.T, nv = H / 8;

  // 1. this warp's router row: all its loads in flight first (weights do not
  //    depend on the previous kernel)
  const int e_row = blockIdx.x * kWarps + warp;
  uint4 gv[kRowChunks];
#pragma unroll
  for (int c = 0; c < kRowChunks; ++c) {
    const int i = c * 256 + lane * 8;
    gv[c] = (e_row < p.E && i < H)
                ? __ldcs(reinterpret_cast<const uint4*>(p.gate_w + size_t(e_row) * H + i))
                : make_uint4(0, 0, 0, 0);
  }
  // this thread's selection biases (stored to shared memory once the
  // tokens are in, so the load does not hold up the wait below)
  const float bias_r =  // (E <= 256 = kThreads)
      p.gate_bias && int(threadIdx.x) < p.E ? __ldg(p.gate_bias + threadIdx.x) : 0.0f;
  pdl_wait();
  // The next launch may start (its prologue overlaps the rest of this
  // kernel) once this kernel's input is complete.
  pdl_trigger();

  // 2. x * w_norm into shared memory (fp32) and the sum of squares per token;
  //    logit_e = r_t * (G_e . (x_t * w)), so the dot products need not wait
  //    for the norm
  float* xw = reinterpret_cast<float*>(dsm);  // [T][H]
  float ss[MAXT];
#pragma unroll
  for (int t = 0; t < MAXT; ++t) ss[t] = 0.f;
  for (int c = threadIdx.x; c < nv; c += kThreads) {
    float g[8];
    unpack8(reinterpret_cast<const uint4*>(p.norm_w)[c], g);
#pragma unroll
    for (int t = 0; t < MAXT; ++t) {
      if (t < T) {
        float f[8];
        unpack8(reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[c], f);
        float* d = xw + t * H + c * 8;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          ss[t] += f[q] * f[q];
          d[q] = f[q] * g[q];
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < MAXT; ++t) {
    const float v = warp_sum(ss[t]);
    if (lane == 0) red[warp][t] = v;
  }
  __syncthreads();
  if (threadIdx.x < T) {
    float v = 0.f;
    for (int w = 0; w < kWarps; ++w) v += red[w][threadIdx.x];
    rs[threadIdx.x] = rsqrtf(v / float(H) + p.eps);
  }
  if (int(threadIdx.x) < p.E) s_bias[threadIdx.x] = bias_r;
  __syncthreads();

  // 3. router logits (fp32) of this warp's expert row
  if (e_row < p.E) {
    float acc[MAXT];
#pragma unroll
    for (int t = 0; t < MAXT; ++t) acc[t] = 0.f;
#pragma unroll
    for (int c = 0; c < kRowChunks; ++c) {
      const int i = c * 256 + lane * 8;
      if (i < H) {
        float gf[8];
        unpack8(gv[c], gf);
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
          if (t < T) {
            const float4 a = *reinterpret_cast<const float4*>(xw + t * H + i);
            const float4 b = *reinterpret_cast<const float4*>(xw + t * H + i + 4);
            acc[t] += gf[0] * a.x + gf[1] * a.y + gf[2] * a.z + gf[3] * a.w + gf[4] * b.x +
                      gf[5] * b.y + gf[6] * b.z + gf[7] * b.w;
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < MAXT; ++t) {
      if (t < T) {
        const float v = warp_sum(acc[t]);
        if (lane == 0) p.ws.logits[t * p.E + e_row] = v * rs[t];
      }
    }
  }
  // block 0: residual copy and the bf16 normed rows the up launch multiplies
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < T * nv; i += kThreads) {
      const int t = i / nv, c = i - t * nv;
      reinterpret_cast<uint4*>(p.residual + size_t(t) * H)[c] =
          reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[c];
      const float* d = xw + t * H + c * 8;
      const float r = rs[t];
      reinterpret_cast<uint4*>(p.ws.x16 + size_t(t) * H)[c] =
          make_uint4(pack_bf16x2(d[0] * r, d[1] * r), pack_bf16x2(d[2] * r, d[3] * r),
                     pack_bf16x2(d[4] * r, d[5] * r), pack_bf16x2(d[6] * r, d[7] * r));
    }
  }

  // ---- the last block to finish routes every token
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) am_last = atomicAdd(p.ws.counter, 1u) == unsigned(gridDim.x - 1);
  __syncthreads();
  if (!am_last) return;
  __threadfence();
  for (int t = warp; t < T; t += kWarps)
    warp_topk(p.ws.logits + t * p.E, p.gate_bias ? s_bias : nullptr, p.E, p.k, p.rsf, s_idx + t * p.k,
              s_w + t * p.k);
  __syncthreads();
  // segments: 0 = shared expert, 1.. = distinct routed experts in first-use
  // order over the pairs f = t*k + j; seg_w[s][t] = routing weight of token t
  // in segment s (0 if not routed to it)
  const int R = T * p.k;
  const int max_slots = R < p.E ? R : p.E;  // segments the workspace holds, minus the shared one
  for (int i = threadIdx.x; i < (max_slots + 1) * kDecodeN; i += kThreads) p.ws.seg_w[i] = 0.f;
  for (int f = threadIdx.x; f < R; f += kThreads) {
    const int e = s_idx[f];
    int first = 1;
    for (int g = 0; g < f; ++g) first &= s_idx[g] != e;
    s_first[f] = first;
    p.ws.idx[f] = e;
    p.ws.w[f] = s_w[f];
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the first-use flags (R <= 128)
    int base = 0;
    for (int f0 = 0; f0 < R; f0 += 32) {
      const int f = f0 + lane;
      const int v = f < R ? s_first[f] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (v) {
        s_seg_of[s_idx[f]] = base + incl - 1;
        s_exp[base + incl - 1] = s_idx[f];
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_nseg = base + 1;
  }
  __syncthreads();
  for (int f = threadIdx.x; f < R; f += kThreads)
    p.ws.seg_w[(s_seg_of[s_idx[f]] + 1) * kDecodeN + f / p.k] = s_w[f];
  const int nseg = s_nseg, nslot = nseg - 1;
  for (int s = threadIdx.x; s < nslot; s += kThreads) p.ws.seg_expert[s + 1] = s_exp[s];
  // up tile list: shared-expert tiles first, then the routed slots, each cut
  // into 128-row tiles (the down launch needs only the segment table)
  const int nI = (p.I + kBM - 1) / kBM, nS = (p.S + kBM - 1) / kBM;
  for (int i = threadIdx.x; i < nS + nslot * nI; i += kThreads) {
    DecodeTile d;
    if (i < nS) {
      d = DecodeTile{1, 0, i * kBM, 0, i * kBM};
    } else {
      const int s = (i - nS) / nI, mt = (i - nS) - s * nI;
      d = DecodeTile{0, s + 1, s_exp[s] * p.I + mt * kBM, 0, mt * kBM};
    }
    p.ws.tiles_up[i] = d;
  }
  if (threadIdx.x == 0) {
    *p.ws.n_tiles_up = nS + nslot * nI;
    *p.ws.n_segments = nseg;
    *p.ws.counter = 0u;
  }
}

size_t route_smem(int T, int H) { return size_t(T) * H * 4; }

constexpr size_t kMaxRouteSmem = 160 * 1024;

}  // namespace

bool decode_supported(const moe_config& c) {
  if (c.latent_size != 0 || c.expert_wdtype != MOE_WEIGHTS_BF16) return false;
  // one router row per warp, held in registers (kRowChunks x 256 elements)
  return c.hidden_size <= kRowChunks * 256 &&
         route_smem(kDecodeMaxT, c.hidden_size) <= kMaxRouteSmem;
}

cudaError_t prepare_decode() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(decode_route<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kMaxRouteSmem))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(decode_route<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kMaxRouteSmem))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(decode_route<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kMaxRouteSmem))) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(decode_route<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(kMaxRouteSmem));
}

cudaError_t launch_decode_route(const DecodeRouteArgs& a, cudaStream_t stream) {
  const moe_config& c = *a.cfg;
  RouteParams rp;
  rp.hidden = a.hidden;
  rp.norm_w = static_cast<const bf16*>(a.w->norm_w);
  rp.gate_w = static_cast<const bf16*>(a.w->gate_w);
  rp.gate_bias = a.w->gate_bias;
  rp.residual = a.residual;
  rp.ws = *a.ws;
  rp.T = a.T;
  rp.H = c.hidden_size;
  rp.E = c.num_experts;
  rp.k = c.top_k;
  rp.I = c.moe_inter;
  rp.S = c.shared_inter;
  rp.eps = c.rms_eps;
  rp.rsf = c.routed_scaling_factor;
  const int blocks = (c.num_experts + kWarps - 1) / kWarps;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = route_smem(a.T, c.hidden_size);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.T <= 1) return cudaLaunchKernelEx(&cfg, decode_route<1>, rp);
  if (a.T <= 2) return cudaLaunchKernelEx(&cfg, decode_route<2>, rp);
  if (a.T <= 4) return cudaLaunchKernelEx(&cfg, decode_route<4>, rp);
  return cudaLaunchKernelEx(&cfg, decode_route<8>, rp);
}

}  // namespace moe
