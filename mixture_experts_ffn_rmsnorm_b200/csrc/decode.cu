// Decode path kernels (1 <= T <= 8 tokens): the layer is weight-streaming
// here, so every kernel is a row-streaming GEMV.  Three launches, chained with
// programmatic dependent launch (each is scheduled while the previous one
// drains; griddepcontrol.wait guards every read of the previous outputs):
//
//   decode_route        blocks [0, G): RMSNorm + FP32 router logits; the last
//                       of them runs a warp-parallel sigmoid top-k per token
//                       and builds the distinct-expert slot table.  Blocks
//                       [G, grid): shared expert up + relu^2 (independent of
//                       routing), and an L2 prefetch of the shared expert's
//                       down weights for the next kernel.
//   decode_up_sdown     routed up + relu^2 for the tokens of every distinct
//                       expert (its weights read once) and the shared expert's
//                       down projection.
//   decode_down_combine every block owns a range of output rows h and streams
//                       those rows of each routed expert's down matrix, then
//                       writes residual + shared + sum_j w_j * y_j (no atomics).
//
// Row streaming: one persistent block per SM.  Lane 0 of warp 0 keeps a
// ring of kStages x 32 KB bulk copies (cp.async.bulk, the TMA's 1-D form) of
// contiguous weight rows in flight; 4 consumer warps take the rows of each
// landed chunk, dot them with the token vectors (L1-resident) and release
// the stage.  Bytes in flight per SM no longer depend on registers.  Every
// mbarrier wait is bounded and records a timeout in the status word.
#include "decode.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kStages = 6;
constexpr int kStageBytes = 32 * 1024;
constexpr int kConsumers = 12;                      // consumer warps
constexpr int kStreamThreads = 32 * (1 + kConsumers);
constexpr int kGateWarps = kConsumers + 1;          // warps of a router block
constexpr int kMaxSlots = kDecodeMaxT * kTopKMax;
constexpr int kRouteStages = 4;                     // decode_route leaves room for token rows

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

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float relu2(float x) { return x > 0.f ? x * x : 0.f; }

// Asynchronously pull `bytes` (multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> shared, completion as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Select v[i] for a runtime i without dynamic register indexing.
template <int N>
__device__ __forceinline__ float pick(const float (&v)[N], int i) {
  float r = 0.f;
#pragma unroll
  for (int j = 0; j < N; ++j)
    if (j == i) r = v[j];
  return r;
}

__device__ __forceinline__ int nt_pad(int n) { return n <= 1 ? 1 : n <= 2 ? 2 : n <= 4 ? 4 : 8; }

// acc[t] = dot(w[0..K), x[t][0..K)) for one row w in shared memory and NT
// token vectors x[t] (generic pointers: global or shared memory, so they are
// read with plain generic loads), reduced across the warp.
template <int NT>
__device__ __forceinline__ void smem_row_dot(const bf16* w, int K, const bf16* const (&x)[NT],
                                             float (&acc)[NT]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t] = 0.f;
#pragma unroll 2
  for (int i = lane * 8; i < K; i += 256) {
    float g[8];
    unpack8(*reinterpret_cast<const uint4*>(w + i), g);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float xf[8];
      unpack8(*reinterpret_cast<const uint4*>(x[t] + i), xf);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[t] = fmaf(g[q], xf[q], acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t] = warp_sum(acc[t]);
}

// ----------------------------------------------------------- stream ring
struct Chunk {
  int seg;     // which matrix family (kernel-specific)
  int slot;    // routed slot (or -1)
  int row0;    // first row inside its matrix
  int nrows;   // rows in the chunk; < 0 = end of stream
};

struct Ring {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  Chunk meta[kStages];
  int nst;    // stages in use (<= kStages)
  int abort;
};

__device__ __forceinline__ uint8_t* ring_buf(uint8_t* dsm, int s) { return dsm + s * kStageBytes; }

__device__ __forceinline__ void ring_init(Ring& r, int nst = kStages) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&r.full[s], 1);
      mbar_init(&r.empty[s], kConsumers);
    }
    r.nst = nst;
    r.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
}

__device__ __forceinline__ void note_timeout(Ring& r, int* status) {
  r.abort = 1;
  if (status) atomicOr(status, kStatusWaitTimeout);
}

// Producer side: state of one lane issuing chunks into the ring.
struct Producer {
  Ring* r;
  uint8_t* dsm;
  int* status;
  int stage = 0;
  uint32_t phase = 0;
  int issued = 0;
  bool ok = true;

  __device__ __forceinline__ void push(const Chunk& c, const void* src, uint32_t bytes) {
    if (!ok) return;
    if (!mbar_wait(&r->empty[stage], phase ^ 1u, &r->abort)) {
      note_timeout(*r, status);
      ok = false;
      return;
    }
    r->meta[stage] = c;
    mbar_arrive_expect_tx(&r->full[stage], bytes);
    bulk_load(ring_buf(dsm, stage), src, bytes, &r->full[stage]);
    ++issued;
    if (++stage == r->nst) {
      stage = 0;
      phase ^= 1u;
    }
  }

  __device__ __forceinline__ void finish() {
    if (ok && mbar_wait(&r->empty[stage], phase ^ 1u, &r->abort)) {
      r->meta[stage] = Chunk{0, -1, 0, -1};
      mbar_arrive(&r->full[stage]);
      return;
    }
    if (ok) note_timeout(*r, status);
    // drain the copies this lane issued before the block exits
    int s = stage;
    uint32_t ph = phase;
    const int n = issued < r->nst ? issued : r->nst;
    for (int i = 0; i < n; ++i) {
      if (--s < 0) {
        s = r->nst - 1;
        ph ^= 1u;
      }
      int zero = 0;
      mbar_wait(&r->full[s], ph, &zero);
    }
  }
};

// Consumer side: iterate the landed chunks until the end marker; f(chunk,
// rows) is called by every consumer warp for each chunk.
template <class F>
__device__ __forceinline__ void consume(Ring& r, uint8_t* dsm, int* status, F f) {
  const int lane = threadIdx.x & 31;
  int stage = 0;
  uint32_t phase = 0;
  while (true) {
    if (!mbar_wait(&r.full[stage], phase, &r.abort)) {
      note_timeout(r, status);
      return;
    }
    const Chunk c = r.meta[stage];
    if (c.nrows < 0) return;
    f(c, reinterpret_cast<const bf16*>(ring_buf(dsm, stage)));
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.empty[stage]);
    if (++stage == r.nst) {
      stage = 0;
      phase ^= 1u;
    }
  }
}

// Push rows [r0, r1) of a row-major [rows, K] bf16 matrix as chunks of at
// most kStageBytes.
__device__ __forceinline__ void push_rows(Producer& pr, int seg, int slot, const bf16* m, int K,
                                          int r0, int r1) {
  const int per = kStageBytes / (K * 2);
  for (int r = r0; r < r1; r += per) {
    const int n = r1 - r < per ? r1 - r : per;
    pr.push(Chunk{seg, slot, r, n}, m + size_t(r) * K, uint32_t(n) * K * 2);
  }
}

// ---------------------------------------------------------------- route
struct RouteParams {
  const bf16* hidden;
  const bf16* norm_w;
  const bf16* gate_w;
  const float* gate_bias;
  const bf16* shared_up_w;
  const void* prefetch;   // shared down weights, prefetched into L2
  size_t prefetch_bytes;
  bf16* residual;
  DecodeWorkspace ws;
  int* status;
  int T, H, E, k, S, gate_blocks;
  float eps, rsf;
};

// Router logits of one expert row for T tokens (fp32 normed input in smem).
__device__ void gate_row(const RouteParams& p, const float* xn, int e) {
  const int lane = threadIdx.x & 31;
  float acc[kDecodeMaxT];
#pragma unroll
  for (int t = 0; t < kDecodeMaxT; ++t) acc[t] = 0.f;
  const bf16* g = p.gate_w + size_t(e) * p.H;
  constexpr int KCH = 16;  // 4096 elements of the row in flight per pass
  for (int k0 = 0; k0 < p.H; k0 += KCH * 256) {
    uint4 wv[KCH];
#pragma unroll
    for (int c = 0; c < KCH; ++c) {
      const int i = k0 + c * 256 + lane * 8;
      wv[c] = i < p.H ? __ldcs(reinterpret_cast<const uint4*>(g + i)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int c = 0; c < KCH; ++c) {
      const int i = k0 + c * 256 + lane * 8;
      if (i < p.H) {
        float gf[8];
        unpack8(wv[c], gf);
#pragma unroll
        for (int t = 0; t < kDecodeMaxT; ++t) {
          if (t < p.T) {
            const float4 a = *reinterpret_cast<const float4*>(xn + t * p.H + i);
            const float4 b = *reinterpret_cast<const float4*>(xn + t * p.H + i + 4);
            acc[t] += gf[0] * a.x + gf[1] * a.y + gf[2] * a.z + gf[3] * a.w + gf[4] * b.x +
                      gf[5] * b.y + gf[6] * b.z + gf[7] * b.w;
          }
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kDecodeMaxT; ++t) {
    if (t < p.T) {
      const float v = warp_sum(acc[t]);
      if (lane == 0) p.ws.logits[t * p.E + e] = v;
    }
  }
}

// Shared expert up rows of one landed chunk: vo[t, row] = bf16(relu^2(n_t . SU[row])).
template <int NT>
__device__ __forceinline__ void shared_up_chunk(const RouteParams& p, const Chunk& c,
                                                const bf16* rows, const bf16* xs) {
  const int warp = (threadIdx.x >> 5) - 1, lane = threadIdx.x & 31;
  const bf16* x[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) x[t] = xs + size_t(t < p.T ? t : 0) * p.H;
  for (int r = warp; r < c.nrows; r += kConsumers) {
    float acc[NT];
    smem_row_dot<NT>(rows + size_t(r) * p.H, p.H, x, acc);
    if (lane < p.T)
      p.ws.vo[size_t(lane) * p.S + c.row0 + r] = __float2bfloat16_rn(relu2(pick(acc, lane)));
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kStreamThreads, 1) decode_route(const RouteParams p) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ Ring ring;
  __shared__ float rs[kDecodeMaxT];
  __shared__ float red[kGateWarps][kDecodeMaxT];
  __shared__ int am_last;
  __shared__ int s_exp[kMaxSlots];
  __shared__ int s_cnt[kMaxSlots];
  __shared__ int s_idx[kMaxSlots];
  __shared__ float s_w[kMaxSlots];
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.H, T = p.T, nv = H / 8;
  const bool router = blockIdx.x < p.gate_blocks;
  if (!router) {
    ring_init(ring, kRouteStages);
    // the shared expert's down weights do not depend on anything: start
    // pulling them into L2 for decode_up_sdown right away
    if (threadIdx.x == 0 && p.prefetch_bytes > 0) {
      const size_t nb = gridDim.x - p.gate_blocks;
      const size_t per = ((p.prefetch_bytes + nb - 1) / nb + 15) & ~size_t(15);
      const size_t b0 = (blockIdx.x - p.gate_blocks) * per;
      const size_t end = b0 + per < p.prefetch_bytes ? b0 + per : p.prefetch_bytes;
      for (size_t o = b0; o < end; o += 65536)
        bulk_prefetch_l2(reinterpret_cast<const char*>(p.prefetch) + o,
                         uint32_t(end - o < 65536 ? end - o : 65536));
    }
  }
  pdl_wait();

  // RMSNorm scale of every token (every block recomputes it; rows are tiny).
  {
    float ss[kDecodeMaxT];
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) ss[t] = 0.f;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
#pragma unroll
      for (int t = 0; t < kDecodeMaxT; ++t) {
        if (t < T) {
          float f[8];
          unpack8(reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[i], f);
#pragma unroll
          for (int q = 0; q < 8; ++q) ss[t] += f[q] * f[q];
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kDecodeMaxT; ++t) {
      const float v = warp_sum(ss[t]);
      if (lane == 0) red[warp][t] = v;
    }
    __syncthreads();
    if (threadIdx.x < T) {
      float v = 0.f;
      for (int w = 0; w < kGateWarps; ++w) v += red[w][threadIdx.x];
      rs[threadIdx.x] = rsqrtf(v / float(H) + p.eps);
    }
    __syncthreads();
  }

  if (!router) {
    // ---- shared expert up projection + relu^2 over bf16(n); the token rows
    // sit right after this kernel's (shorter) ring in dynamic shared memory
    bf16* xs = reinterpret_cast<bf16*>(dsm + size_t(kRouteStages) * kStageBytes);
    for (int i = threadIdx.x; i < T * nv; i += blockDim.x) {
      const int t = i / nv, c = i - t * nv;
      float f[8], g[8];
      unpack8(reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[c], f);
      unpack8(reinterpret_cast<const uint4*>(p.norm_w)[c], g);
      const float r = rs[t];
      reinterpret_cast<uint4*>(xs + size_t(t) * H)[c] =
          make_uint4(pack_bf16x2(f[0] * r * g[0], f[1] * r * g[1]),
                     pack_bf16x2(f[2] * r * g[2], f[3] * r * g[3]),
                     pack_bf16x2(f[4] * r * g[4], f[5] * r * g[5]),
                     pack_bf16x2(f[6] * r * g[6], f[7] * r * g[7]));
    }
    __syncthreads();
    const int nb = gridDim.x - p.gate_blocks, b = blockIdx.x - p.gate_blocks;
    const int r0 = int(int64_t(p.S) * b / nb), r1 = int(int64_t(p.S) * (b + 1) / nb);
    if (warp == 0) {
      if (lane == 0) {
        Producer pr{&ring, dsm, p.status};
        push_rows(pr, 0, -1, p.shared_up_w, H, r0, r1);
        pr.finish();
      }
    } else {
      consume(ring, dsm, p.status, [&](const Chunk& c, const bf16* rows) {
        switch (nt_pad(T)) {
          case 1: shared_up_chunk<1>(p, c, rows, xs); break;
          case 2: shared_up_chunk<2>(p, c, rows, xs); break;
          case 4: shared_up_chunk<4>(p, c, rows, xs); break;
          default: shared_up_chunk<8>(p, c, rows, xs); break;
        }
      });
    }
    return;
  }

  // ---- router logits in float32 from the un-rounded normed vector
  float* xn = reinterpret_cast<float*>(dsm);  // [T][H]
  for (int i = threadIdx.x; i < T * nv; i += blockDim.x) {
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
      reinterpret_cast<uint4*>(p.ws.normed + size_t(t) * H)[c] =
          make_uint4(pack_bf16x2(d[0], d[1]), pack_bf16x2(d[2], d[3]),
                     pack_bf16x2(d[4], d[5]), pack_bf16x2(d[6], d[7]));
    }
  }
  __syncthreads();
  for (int e = blockIdx.x * kGateWarps + warp; e < p.E; e += p.gate_blocks * kGateWarps)
    gate_row(p, xn, e);

  // ---- the last router block to finish routes every token
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) am_last = atomicAdd(p.ws.counter, 1u) == unsigned(p.gate_blocks - 1);
  __syncthreads();
  if (!am_last) return;
  __threadfence();
  for (int t = warp; t < T; t += kGateWarps) {
    warp_topk(p.ws.logits + t * p.E, p.gate_bias, p.E, p.k, p.rsf, s_idx + t * p.k,
              s_w + t * p.k);
    __syncwarp();
    if (lane < p.k) {
      p.ws.idx[t * p.k + lane] = s_idx[t * p.k + lane];
      p.ws.w[t * p.k + lane] = s_w[t * p.k + lane];
    }
  }
  __syncthreads();
  if (warp == 0) {
    // Distinct experts in first-use order, each with its (token, pair,
    // weight) list; pairs are visited in (token, slot) order.
    int n = 0;
    for (int f = 0; f < T * p.k; ++f) {
      const int e = s_idx[f];
      int slot = n;
      for (int base = 0; base < n; base += 32) {
        const unsigned m = __ballot_sync(0xffffffffu, base + lane < n && s_exp[base + lane] == e);
        if (m) {
          slot = base + __ffs(m) - 1;
          break;
        }
      }
      if (slot == n) {
        if (lane == 0) {
          s_exp[n] = e;
          s_cnt[n] = 0;
        }
        ++n;
      }
      __syncwarp();
      if (lane == 0) {
        const int j = s_cnt[slot]++;
        p.ws.slot_tok[slot * kDecodeMaxT + j] = f / p.k;
        p.ws.slot_pair[slot * kDecodeMaxT + j] = f;
        p.ws.slot_w[slot * kDecodeMaxT + j] = s_w[f];
      }
      __syncwarp();
    }
    for (int s = lane; s < n; s += 32) {
      p.ws.slot_expert[s] = s_exp[s];
      p.ws.slot_cnt[s] = s_cnt[s];
    }
    if (lane == 0) {
      *p.ws.n_slots = n;
      *p.ws.counter = 0u;
    }
  }
}

// ------------------------------------------------------ slot table cache
struct SlotCache {
  int n;
  int exp[kMaxSlots];
  int cnt[kMaxSlots];
  int tok[kMaxSlots * kDecodeMaxT];
  int pair[kMaxSlots * kDecodeMaxT];
  float w[kMaxSlots * kDecodeMaxT];
};

__device__ __forceinline__ void load_slots(const DecodeWorkspace& ws, SlotCache& c) {
  const int n = *ws.n_slots;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    c.exp[i] = ws.slot_expert[i];
    c.cnt[i] = ws.slot_cnt[i];
  }
  for (int i = threadIdx.x; i < n * kDecodeMaxT; i += blockDim.x) {
    c.tok[i] = ws.slot_tok[i];
    c.pair[i] = ws.slot_pair[i];
    c.w[i] = ws.slot_w[i];
  }
  if (threadIdx.x == 0) c.n = n;
  __syncthreads();
}

// ------------------------------------------------- routed up + shared down
struct UpParams {
  const bf16* up_w;           // [E, I, H]
  const bf16* shared_down_w;  // [H, S]
  DecodeWorkspace ws;
  int* status;
  int T, H, I, S;
};

template <int NT>
__device__ __forceinline__ void routed_up_chunk(const UpParams& p, const SlotCache& sc,
                                                const Chunk& c, const bf16* rows) {
  const int warp = (threadIdx.x >> 5) - 1, lane = threadIdx.x & 31;
  const int cnt = sc.cnt[c.slot];
  const bf16* x[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t)
    x[t] = p.ws.normed + size_t(sc.tok[c.slot * kDecodeMaxT + (t < cnt ? t : 0)]) * p.H;
  const int pair = lane < cnt ? sc.pair[c.slot * kDecodeMaxT + lane] : 0;
  for (int r = warp; r < c.nrows; r += kConsumers) {
    float acc[NT];
    smem_row_dot<NT>(rows + size_t(r) * p.H, p.H, x, acc);
    if (lane < cnt)
      p.ws.uo[size_t(pair) * p.I + c.row0 + r] = __float2bfloat16_rn(relu2(pick(acc, lane)));
  }
}

template <int NT>
__device__ __forceinline__ void shared_down_chunk(const UpParams& p, const Chunk& c,
                                                  const bf16* rows) {
  const int warp = (threadIdx.x >> 5) - 1, lane = threadIdx.x & 31;
  const bf16* x[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) x[t] = p.ws.vo + size_t(t < p.T ? t : 0) * p.S;
  for (int r = warp; r < c.nrows; r += kConsumers) {
    float acc[NT];
    smem_row_dot<NT>(rows + size_t(r) * p.S, p.S, x, acc);
    if (lane < p.T) p.ws.sh[size_t(lane) * p.H + c.row0 + r] = pick(acc, lane);
  }
}

__global__ void __launch_bounds__(kStreamThreads, 1) decode_up_sdown(const UpParams p) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ Ring ring;
  __shared__ SlotCache sc;
  pdl_trigger();
  ring_init(ring);
  pdl_wait();
  load_slots(p.ws, sc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this block's share of the bytes of [routed up rows | shared down rows]
  const int64_t rb0 = int64_t(p.H) * 2, rb1 = int64_t(p.S) * 2;
  const int64_t n0 = int64_t(sc.n) * p.I, tot0 = n0 * rb0, tot = tot0 + int64_t(p.H) * rb1;
  const int64_t sb = tot * blockIdx.x / gridDim.x, eb = tot * (blockIdx.x + 1) / gridDim.x;
  const int64_t sa = sb < tot0 ? sb : tot0, ea = eb < tot0 ? eb : tot0;
  const int64_t ss2 = sb > tot0 ? sb - tot0 : 0, es2 = eb > tot0 ? eb - tot0 : 0;
  const int64_t a0 = (sa + rb0 - 1) / rb0, a1 = (ea + rb0 - 1) / rb0;
  const int64_t b0 = (ss2 + rb1 - 1) / rb1, b1 = (es2 + rb1 - 1) / rb1;
  if (warp == 0) {
    if (lane == 0) {
      Producer pr{&ring, dsm, p.status};
      for (int64_t r = a0; r < a1;) {  // routed rows, never crossing a slot
        const int slot = int(r / p.I), i0 = int(r - int64_t(slot) * p.I);
        const int64_t left = a1 - r;
        const int i1 = left < int64_t(p.I - i0) ? int(i0 + left) : p.I;
        push_rows(pr, 0, slot, p.up_w + size_t(sc.exp[slot]) * p.I * p.H, p.H, i0, i1);
        r += i1 - i0;
      }
      push_rows(pr, 1, -1, p.shared_down_w, p.S, int(b0), int(b1));
      pr.finish();
    }
  } else {
    const int ntall = nt_pad(p.T);
    consume(ring, dsm, p.status, [&](const Chunk& c, const bf16* rows) {
      if (c.seg == 0) {
        switch (nt_pad(sc.cnt[c.slot])) {
          case 1: routed_up_chunk<1>(p, sc, c, rows); break;
          case 2: routed_up_chunk<2>(p, sc, c, rows); break;
          case 4: routed_up_chunk<4>(p, sc, c, rows); break;
          default: routed_up_chunk<8>(p, sc, c, rows); break;
        }
      } else {
        switch (ntall) {
          case 1: shared_down_chunk<1>(p, c, rows); break;
          case 2: shared_down_chunk<2>(p, c, rows); break;
          case 4: shared_down_chunk<4>(p, c, rows); break;
          default: shared_down_chunk<8>(p, c, rows); break;
        }
      }
    });
  }
}

// ------------------------------------------- routed down + weighted combine
struct DownParams {
  const bf16* down_w;  // [E, H, I]
  const bf16* residual;
  bf16* hidden;
  DecodeWorkspace ws;
  int* status;
  int T, H, I;
};

constexpr int kMaxRowsPerBlock = 64;

// out[h - h0][token] += w * (W_down[e][h] . uo[pair]) for the rows of one
// chunk; a row is always handled by the warp (h - h0) % kConsumers, so each
// accumulator has a single writer.
template <int NT>
__device__ __forceinline__ void down_chunk(const DownParams& p, const SlotCache& sc,
                                           const Chunk& c, const bf16* rows, int h0,
                                           float (*out)[kDecodeMaxT]) {
  const int warp = (threadIdx.x >> 5) - 1, lane = threadIdx.x & 31;
  const int s = c.slot, cnt = sc.cnt[s];
  const bf16* x[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t)
    x[t] = p.ws.uo + size_t(sc.pair[s * kDecodeMaxT + (t < cnt ? t : 0)]) * p.I;
  int r = (warp - (c.row0 - h0)) % kConsumers;
  if (r < 0) r += kConsumers;
  for (; r < c.nrows; r += kConsumers) {
    float acc[NT];
    smem_row_dot<NT>(rows + size_t(r) * p.I, p.I, x, acc);
    if (lane == 0) {
      float* o = out[c.row0 + r - h0];
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (t < cnt) o[sc.tok[s * kDecodeMaxT + t]] += sc.w[s * kDecodeMaxT + t] * acc[t];
    }
  }
}

__global__ void __launch_bounds__(kStreamThreads, 1) decode_down_combine(const DownParams p) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ Ring ring;
  __shared__ SlotCache sc;
  __shared__ float out[kMaxRowsPerBlock][kDecodeMaxT];
  pdl_trigger();
  ring_init(ring);
  for (int i = threadIdx.x; i < kMaxRowsPerBlock * kDecodeMaxT; i += blockDim.x)
    (&out[0][0])[i] = 0.f;
  pdl_wait();
  load_slots(p.ws, sc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h0 = int(int64_t(p.H) * blockIdx.x / gridDim.x);
  const int h1 = int(int64_t(p.H) * (blockIdx.x + 1) / gridDim.x);
  if (warp == 0) {
    if (lane == 0) {
      Producer pr{&ring, dsm, p.status};
      for (int s = 0; s < sc.n; ++s)
        push_rows(pr, 0, s, p.down_w + size_t(sc.exp[s]) * p.H * p.I, p.I, h0, h1);
      pr.finish();
    }
  } else {
    consume(ring, dsm, p.status, [&](const Chunk& c, const bf16* rows) {
      switch (nt_pad(sc.cnt[c.slot])) {
        case 1: down_chunk<1>(p, sc, c, rows, h0, out); break;
        case 2: down_chunk<2>(p, sc, c, rows, h0, out); break;
        case 4: down_chunk<4>(p, sc, c, rows, h0, out); break;
        default: down_chunk<8>(p, sc, c, rows, h0, out); break;
      }
    });
  }
  __syncthreads();
  for (int i = threadIdx.x; i < (h1 - h0) * p.T; i += blockDim.x) {
    const int r = i / p.T, t = i - r * p.T;
    const size_t o = size_t(t) * p.H + h0 + r;
    const float v = __bfloat162float(p.residual[o]) + p.ws.sh[o] + out[r][t];
    p.hidden[o] = __float2bfloat16_rn(v);
  }
}

constexpr size_t kRingBytes = size_t(kStages) * kStageBytes;

template <class Kern, class Params>
cudaError_t launch_pdl(Kern k, dim3 grid, size_t smem, cudaStream_t s, const Params& prm) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kStreamThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, prm);
}

// decode_route's dynamic shared memory: the ring plus the bf16 token rows
// (streaming blocks), or the fp32 token rows (router blocks).
size_t route_smem(int T, int H) {
  const size_t a = size_t(kRouteStages) * kStageBytes + size_t(T) * H * 2, b = size_t(T) * H * 4;
  return a > b ? a : b;
}

constexpr size_t kMaxDynSmem = 227 * 1024 - 20 * 1024;  // leave room for the static arrays

}  // namespace

bool decode_supported(const moe_config& c) {
  if (c.latent_size != 0 || c.expert_wdtype != MOE_WEIGHTS_BF16) return false;
  // a weight row must fit one ring stage; the token rows must fit next to the ring
  const int maxk = c.hidden_size > c.moe_inter
                       ? (c.hidden_size > c.shared_inter ? c.hidden_size : c.shared_inter)
                       : (c.moe_inter > c.shared_inter ? c.moe_inter : c.shared_inter);
  return size_t(maxk) * 2 <= size_t(kStageBytes) &&
         route_smem(kDecodeMaxT, c.hidden_size) <= kMaxDynSmem;
}

cudaError_t prepare_decode() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(decode_route, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kMaxDynSmem))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(decode_up_sdown, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(kRingBytes))) != cudaSuccess)
    return e;
  return cudaFuncSetAttribute(decode_down_combine, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(kRingBytes));
}

moe_status enqueue_decode(const DecodeArgs& a, bf16* hidden, bf16* residual, int T,
                          cudaStream_t stream, LaunchLog* log) {
  const moe_config& c = *a.cfg;
  if (!decode_supported(c) || T < 1 || T > kDecodeMaxT) return MOE_ERR_INVALID_CONFIG;
  const int H = c.hidden_size, E = c.num_experts, k = c.top_k, I = c.moe_inter,
            S = c.shared_inter;
  const int sms = a.num_sms > 0 ? a.num_sms : 148;

  RouteParams rp;
  rp.hidden = hidden;
  rp.norm_w = static_cast<const bf16*>(a.w->norm_w);
  rp.gate_w = static_cast<const bf16*>(a.w->gate_w);
  rp.gate_bias = a.w->gate_bias;
  rp.shared_up_w = static_cast<const bf16*>(a.w->shared_up_w);
  rp.prefetch = a.w->shared_down_w;
  rp.prefetch_bytes = size_t(H) * S * 2;
  rp.residual = residual;
  rp.ws = *a.ws;
  rp.status = a.status;
  rp.T = T;
  rp.H = H;
  rp.E = E;
  rp.k = k;
  rp.S = S;
  rp.gate_blocks = (E + kGateWarps - 1) / kGateWarps;
  if (rp.gate_blocks > sms / 4) rp.gate_blocks = sms / 4 > 0 ? sms / 4 : 1;
  rp.eps = c.rms_eps;
  rp.rsf = c.routed_scaling_factor;
  const int sblocks = sms - rp.gate_blocks > 1 ? sms - rp.gate_blocks : 1;
  if (launch_pdl(decode_route, dim3(rp.gate_blocks + sblocks), route_smem(T, H), stream, rp) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  log->done(stream);

  UpParams up;
  up.up_w = static_cast<const bf16*>(a.w->up_w);
  up.shared_down_w = static_cast<const bf16*>(a.w->shared_down_w);
  up.ws = *a.ws;
  up.status = a.status;
  up.T = T;
  up.H = H;
  up.I = I;
  up.S = S;
  if (launch_pdl(decode_up_sdown, dim3(sms), kRingBytes, stream, up) != cudaSuccess)
    return MOE_ERR_CUDA;
  log->done(stream);

  DownParams dp;
  dp.down_w = static_cast<const bf16*>(a.w->down_w);
  dp.residual = residual;
  dp.hidden = hidden;
  dp.ws = *a.ws;
  dp.status = a.status;
  dp.T = T;
  dp.H = H;
  dp.I = I;
  int dblocks = sms;
  if (dblocks > H) dblocks = H;
  while ((H + dblocks - 1) / dblocks > kMaxRowsPerBlock) ++dblocks;
  if (launch_pdl(decode_down_combine, dim3(dblocks), kRingBytes, stream, dp) != cudaSuccess)
    return MOE_ERR_CUDA;
  log->done(stream);
  return MOE_OK;
}

}  // namespace moe
