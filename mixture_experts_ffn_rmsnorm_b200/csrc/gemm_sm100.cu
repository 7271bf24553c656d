// Persistent grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
// The grouped up- and down-projections of the routed experts (MoeLayer,
// `forward_prefill`: sort-by-expert, then a tensor-core GEMM per expert with
// each expert's weights loaded once), run together with a dense "class" of
// tiles in the same launch (the always-on shared expert, nemotron_moe.rs
// `prefill`, or LatentMoE fc1 / fc2), and the router GEMM with the sigmoid
// top-k routing fused into its epilogue (or, with K split over idle SMs,
// storing fp32 partial logits for the reduction kernel).  The grouped up and
// down launches take their tiles dynamically from a device counter; the
// router and fc2 launches walk a static round-robin.
//
// Structure (one CTA per SM, persistent over its tiles):
//   warp 0   one lane issues TMA loads of A (128 x 128 B) and B (BN x 128 B)
//            K-blocks into a STAGES-deep shared-memory ring (128-byte swizzle);
//   warp 1   owns TMEM (2 x BN fp32 columns = two accumulators) and one lane
//            issues tcgen05.mma (M = 128, N = BN) per K-step, committing each
//            stage back to the producer and each finished tile to the epilogue;
//   warps 2-5 read the accumulator rows from TMEM (tcgen05.ld), apply the
//            epilogue (relu^2, scales, top-k, blend) and store to global
//            memory while the MMA warp fills the other accumulator.
// Every wait is bounded: a timeout sets a status bit and the CTA winds down
// (draining its own TMA loads and MMAs) instead of hanging.
#include "moe_internal.h"
#include "ptx.cuh"
#include "topk.cuh"
#include "../../include/moe_b200.h"

namespace moe {
namespace {

// A stage holds 128 bytes of K per row for both operand types: 64 BF16 or
// 128 E4M3 elements; one tcgen05.mma consumes 32 bytes of K (16 BF16 or
// 32 E4M3), so the smem layout and descriptors are type independent.
template <int BN, int STAGES>
struct Traits {
  static constexpr int kABytes = kBM * 128;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kKSteps = 4;                 // 4 x 32 bytes of K per stage
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kSmem = STAGES * kStageBytes + 1024 + 512;
  static_assert(kTmemCols == 256 || kTmemCols == 512,
                "TMEM allocation must be a power of two >= 32");
};

__device__ __forceinline__ int stage_k(const GemmClass& C) { return C.fp8 ? 128 : 64; }

struct Tile {
  int c;        // class
  int e;        // group (expert) index
  int row0;     // first A row
  int row_end;  // first row not stored
  int n0;       // first output column
  int brow;     // first B row
  int arow;     // first A row to load
  int split;    // K split index (dense classes)
  int k0, k1;   // K-block range [k0, k1); k1 < 0 = through the end
};

// Tile number w of the launch: class 0 (routed groups through the m-tile
// table, or a dense class with its K splits) for w < W0, then class 1.
template <int BN>
__device__ __forceinline__ Tile tile_at(const GemmParams& p, int w, int W0) {
  Tile t;
  t.split = 0;
  t.k0 = 0;
  t.k1 = -1;
  if (w < W0) {
    const int ks = p.cls[0].ksplit > 1 ? p.cls[0].ksplit : 1;
    const int nt = p.cls[0].ntiles * ks;
    const int mt = w / nt;
    int ni = w - mt * nt;
    if (ks > 1) {
      t.split = ni % ks;
      ni /= ks;
      const int bk = p.cls[0].fp8 ? 128 : 64;
      const int nk = (p.cls[0].K + bk - 1) / bk;
      const int per = (nk + ks - 1) / ks;
      t.k0 = t.split * per;
      t.k1 = min(nk, t.k0 + per);
    }
    t.c = 0;
    if (p.tile_table) {
      const int2 te = p.tile_table[mt];
      t.e = te.x;
      t.row0 = te.y;
      t.row_end = p.group_off[te.x + 1];
    } else {
      t.e = 0;
      t.row0 = mt * kBM;
      t.row_end = p.cls[0].rows;
    }
    t.n0 = ni * BN;
  } else {
    w -= W0;
    const int nt = p.cls[1].ntiles;
    const int mt = w / nt;
    const int ni = w - mt * nt;
    t.c = 1;
    t.e = 0;
    t.row0 = mt * kBM;
    t.row_end = p.cls[1].rows;
    t.n0 = ni * BN;
  }
  t.brow = t.e * p.cls[t.c].N + t.n0;
  t.arow = t.row0;
  return t;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
    u.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
    u.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
    u.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
    d[i] = u;
  }
}

// The it-th tile of this CTA in the static schedule: tile blockIdx.x +
// it * gridDim.x.
template <int BN>
__device__ __forceinline__ bool work_item(const GemmParams& p, int W, int W0, int it, Tile* t) {
  const int w = int(blockIdx.x) + it * int(gridDim.x);
  if (w >= W) return false;
  *t = tile_at<BN>(p, w, W0);
  return true;
}

// Dynamic schedule: the producer publishes each tile index through a ring
// of kTileRing slots that the MMA thread and the four epilogue warps read in
// the same order.
constexpr int kTileRing = 8;

// Order of the dynamically handed-out tiles: the shared class (class 1,
// whose tiles have the longer K) first, so that the short routed tiles
// fill the end of the launch.
__device__ __forceinline__ int dyn_tile_index(int j, int W0, int W) {
  const int W1 = W - W0;
  return j < W1 ? W0 + j : j - W1;
}

__device__ __forceinline__ void record_timeout(const GemmParams& p, volatile int* abort) {
  *abort = 1;
  if (p.status) atomicOr(p.status, kStatusWaitTimeout);
}

// Router epilogue: one thread per token row holds its E <= BN logits.
// Without split K the thread runs the sigmoid top-k itself and the tile's
// expert histogram (for the sort) is accumulated in shared memory and
// written out.  With split K every split only stores its fp32 partial
// logits, row-major [split][row][E], for the reduction kernel.
template <int BN>
__device__ __forceinline__ void router_epilogue(const GemmParams& p, const GemmClass& C,
                                                const Tile& t, uint32_t tb, int row,
                                                bool rvalid) {
  __shared__ int s_hist[MOE_MAX_EXPERTS];
  const int E = p.num_experts;
  const int ep = threadIdx.x - 2 * 32;  // 0..127 inside the epilogue warps
  if (C.ksplit > 1) {
    float* prow = p.topk_part + (size_t(t.split) * p.topk_rows_cap + row) * E;
    const bool vec = (E & 3) == 0;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tb + uint32_t(c * 32), r);
      tmem_ld_wait();
      if (rvalid) {
        if (vec) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            if (c * 32 + j < E)
              *reinterpret_cast<float4*>(prow + c * 32 + j) =
                  make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                              __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j < E) prow[c * 32 + j] = __uint_as_float(r[j]);
        }
      }
    }
    return;
  }
  TopK tk;
  tk.init();
  // the accumulator holds G' . x; the token's factor makes it the logits
  const float rsc = p.topk_rs && rvalid ? p.topk_rs[row] : 1.f;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tb + uint32_t(c * 32), r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int e = c * 32 + j;
      if (e < E)
        tk.offer(e, __uint_as_float(r[j]) * rsc, p.gate_bias ? p.gate_bias[e] : 0.0f, p.top_k);
    }
  }
  const int mt = t.row0 / kBM;
  for (int e = ep; e < E; e += 4 * 32) s_hist[e] = 0;
  named_barrier(1, 4 * 32);
  if (rvalid) {
    tk.write(p.top_k, p.rsf, p.topk_idx + size_t(row) * p.top_k, p.topk_w + size_t(row) * p.top_k);
#pragma unroll
    for (int j = 0; j < kTopKMax; ++j)  // (an unfilled slot, id -1, only with NaN logits)
      if (j < p.top_k && unsigned(tk.id[j]) < unsigned(E)) atomicAdd(&s_hist[tk.id[j]], 1);
  }
  named_barrier(1, 4 * 32);
  if (p.expert_hist)
    for (int e = ep; e < E; e += 4 * 32) p.expert_hist[size_t(mt) * E + e] = s_hist[e];
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  using Tr = Traits<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* tiles = smem_raw + pad;
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + STAGES * Tr::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* rfull = drain + 2;  // tile-index ring (dynamic schedule)
  uint64_t* rempty = rfull + kTileRing;
  volatile int* ring = reinterpret_cast<volatile int*>(rempty + kTileRing);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < kTileRing; ++s) {
      mbar_init(&rfull[s], 1);
      mbar_init(&rempty[s], 5);  // the MMA thread and the four epilogue warps
    }
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA[0]);
    tma_prefetch_desc(&p.tmB[0]);
    if (p.nclasses > 1) {
      tma_prefetch_desc(&p.tmA[1]);
      tma_prefetch_desc(&p.tmB[1]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Tr::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above overlaps the previous kernel when launched with PDL.
  // Dependents may start once every CTA is past this point.  With epi_wait
  // the producer and the MMA warp go on at once (their operands do not
  // depend on the previous kernel) and only the epilogue warps wait; every
  // CTA still waits before it exits, so the launch completes after the
  // previous one.
  if (!p.epi_wait || warp >= 2) pdl_wait();
  pdl_trigger();

  const int m0 = p.n_mtiles ? *p.n_mtiles : p.cls[0].mtiles;
  const int W0 = m0 * p.cls[0].ntiles * (p.cls[0].ksplit > 1 ? p.cls[0].ksplit : 1);
  const int W = W0 + (p.nclasses > 1 ? p.cls[1].mtiles * p.cls[1].ntiles : 0);
  const bool dyn = p.sched != nullptr;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      // dynamic schedule: the next tile (the first is blockIdx.x) is taken
      // from the counter two k-blocks before the current tile's last load
      int nxt = int(blockIdx.x);
      bool fetched = true;
      for (int it = 0; ok; ++it) {
        Tile t;
        if (dyn) {
          const int slot = it & (kTileRing - 1);
          if (!mbar_wait(&rempty[slot], ((it / kTileRing) & 1) ^ 1u, abort)) {
            record_timeout(p, abort);
            break;
          }
          const int w = nxt < W ? dyn_tile_index(nxt, W0, W) : -1;
          ring[slot] = w;
          mbar_arrive(&rfull[slot]);
          if (w < 0) break;
          t = tile_at<BN>(p, w, W0);
          fetched = false;
        } else if (!work_item<BN>(p, W, W0, it, &t)) {
          break;
        }
        const GemmClass& C = p.cls[t.c];
        const int bk = stage_k(C);
        const int nk = t.k1 >= 0 ? t.k1 : (C.K + bk - 1) / bk;
        const int fetch_kb = nk - 2 > t.k0 ? nk - 2 : t.k0;
        for (int kb = t.k0; kb < nk; ++kb) {
          if (!fetched && kb == fetch_kb) {
            nxt = int(gridDim.x) + atomicAdd(p.sched, 1);
            fetched = true;
          }
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort)) {
            record_timeout(p, abort);
            ok = false;
            break;
          }
          uint8_t* sa = tiles + stage * Tr::kStageBytes;
          uint8_t* sb = sa + Tr::kABytes;
          mbar_arrive_expect_tx(&full[stage], Tr::kStageBytes);
          const int kx = kb * bk;
          const int kax = C.a_kwrap ? (kx % C.a_kwrap) : kx;
          const int kbx = C.b_kwrap ? (kx % C.b_kwrap) : kx;
          tma_load_2d(sa, &p.tmA[t.c], &full[stage], kax, t.arow);
          tma_load_2d(sb, &p.tmB[t.c], &full[stage], kbx, t.brow);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok && !fetched) {
          nxt = int(gridDim.x) + atomicAdd(p.sched, 1);
          fetched = true;
        }
      }
      if (!ok) {
        // Let the loads this thread issued land before the CTA exits: wait
        // (bounded, ignoring the abort flag) on the last min(issued, STAGES)
        // full barriers.
        int s = stage;
        uint32_t ph = phase;
        const int n = issued < STAGES ? issued : STAGES;
        for (int i = 0; i < n; ++i) {
          if (--s < 0) {
            s = STAGES - 1;
            ph ^= 1u;
          }
          int zero = 0;
          mbar_wait(&full[s], ph, &zero);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_f16 = make_idesc(kBM, BN, 1, 1);  // BF16 x BF16 -> F32
      const uint32_t idesc_f8 = make_idesc(kBM, BN, 0, 0);   // E4M3 x E4M3 -> F32
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        Tile t;
        if (dyn) {
          const int slot = it & (kTileRing - 1);
          if (!mbar_wait(&rfull[slot], (it / kTileRing) & 1, abort)) {
            record_timeout(p, abort);
            break;
          }
          const int w = ring[slot];
          mbar_arrive(&rempty[slot]);
          if (w < 0) break;
          t = tile_at<BN>(p, w, W0);
        } else if (!work_item<BN>(p, W, W0, it, &t)) {
          break;
        }
        const bool f8 = p.cls[t.c].fp8 != 0;
        const int bk = f8 ? 128 : 64;
        const int nk = t.k1 >= 0 ? t.k1 : (p.cls[t.c].K + bk - 1) / bk;
        const int ab = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[ab], aph ^ 1u, abort)) {
          record_timeout(p, abort);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(ab * BN);
        for (int kb = t.k0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort)) {
            record_timeout(p, abort);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* sa = tiles + stage * Tr::kStageBytes;
          const uint64_t ad = smem_desc_sw128(sa);
          const uint64_t bd = smem_desc_sw128(sa + Tr::kABytes);
#pragma unroll
          for (int kk = 0; kk < Tr::kKSteps; ++kk) {
            const uint64_t koff = uint64_t((kk * 32) >> 4);
            const uint32_t acc = (kb != t.k0 || kk != 0) ? 1u : 0u;
            if (f8)
              umma_f8(d, ad + koff, bd + koff, idesc_f8, acc);
            else
              umma_f16(d, ad + koff, bd + koff, idesc_f16, acc);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[ab]);
      }
      // All MMAs this thread issued have completed once `drain` flips.
      umma_commit(drain);
      int zero = 0;
      mbar_wait(drain, 0, &zero);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int rloc = q * 32 + lane;
    for (int it = 0;; ++it) {
      Tile t;
      if (dyn) {  // lane 0 takes the index from the ring for the warp
        const int slot = it & (kTileRing - 1);
        int w = -1, got = 1;
        if (lane == 0) {
          got = mbar_wait(&rfull[slot], (it / kTileRing) & 1, abort);
          if (got) {
            w = ring[slot];
            mbar_arrive(&rempty[slot]);
          } else {
            record_timeout(p, abort);
          }
        }
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!__shfl_sync(0xffffffffu, got, 0) || w < 0) break;
        t = tile_at<BN>(p, w, W0);
      } else if (!work_item<BN>(p, W, W0, it, &t)) {
        break;
      }
      const GemmClass& C = p.cls[t.c];
      const int ab = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!mbar_wait(&tfull[ab], aph, abort)) {
        record_timeout(p, abort);
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(ab * BN);
      const int row = t.row0 + rloc;
      const bool rvalid = row < t.row_end;

      if (C.epi == EPI_TOPK) {
        router_epilogue<BN>(p, C, t, tb, row, rvalid);
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tb + uint32_t(c * 32), r);
          tmem_ld_wait();
          const int n = t.n0 + c * 32;
          if (rvalid && n < C.N) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            if (C.col_scale) {
              const float4* cs =
                  reinterpret_cast<const float4*>(C.col_scale + size_t(t.e) * C.N + n);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float4 s4 = cs[j];
                v[4 * j + 0] *= s4.x;
                v[4 * j + 1] *= s4.y;
                v[4 * j + 2] *= s4.z;
                v[4 * j + 3] *= s4.w;
              }
            }
            if (C.row_scale) {
              const float rs = C.row_scale[row];
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] *= rs;
            }
            if (C.epi == EPI_RELU2_BF16) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = v[j] > 0.f ? v[j] * v[j] : 0.f;
              if (C.row_amax) {
                float m = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) m = fmaxf(m, v[j]);
                atomicMax(C.row_amax + row, __float_as_uint(m));
              }
            }
            if (C.epi == EPI_F32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(C.out) +
                                                      size_t(row) * C.ldo + n);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            } else {
              if (C.epi == EPI_BLEND) {
                const float4* s4 =
                    reinterpret_cast<const float4*>(p.blend_s + size_t(row) * C.ldo + n);
                const uint4* r4 =
                    reinterpret_cast<const uint4*>(p.blend_res + size_t(row) * C.ldo + n);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float4 a = s4[j];
                  v[4 * j + 0] += a.x;
                  v[4 * j + 1] += a.y;
                  v[4 * j + 2] += a.z;
                  v[4 * j + 3] += a.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const uint4 u = r4[j];
                  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                  for (int h = 0; h < 4; ++h) {
                    v[8 * j + 2 * h] += __uint_as_float(w4[h] << 16);
                    v[8 * j + 2 * h + 1] += __uint_as_float(w4[h] & 0xFFFF0000u);
                  }
                }
              }
              store_bf16x32(static_cast<__nv_bfloat16*>(C.out) + size_t(row) * C.ldo + n, v);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Tr::kTmemCols);
  }
  if (dyn && threadIdx.x == 0) {
    // every producer of the grid has taken its last index once all CTAs
    // have counted themselves out: the last one zeroes the counters
    __threadfence();
    if (atomicAdd(p.sched + 1, 1) == int(gridDim.x) - 1) {
      atomicExch(p.sched, 0);
      atomicExch(p.sched + 1, 0);
    }
  }
}

template <int BN, int STAGES>
cudaError_t launch_impl(const GemmParams& p, int grid, cudaStream_t stream, bool pdl) {
  using Tr = Traits<BN, STAGES>;
  if (grid <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = Tr::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<BN, STAGES>, p);
}

template <int BN, int STAGES>
cudaError_t prepare_impl() {
  using Tr = Traits<BN, STAGES>;
  return cudaFuncSetAttribute(grouped_gemm_kernel<BN, STAGES>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::kSmem);
}

}  // namespace

cudaError_t prepare_grouped_gemm() {
  cudaError_t e;
  if ((e = prepare_impl<128, 6>()) != cudaSuccess) return e;
  return prepare_impl<256, 4>();
}

cudaError_t launch_grouped_gemm(const GemmParams& p, int bn, int grid, cudaStream_t stream,
                                bool pdl) {
  if (bn == 128) return launch_impl<128, 6>(p, grid, stream, pdl);
  if (bn == 256) return launch_impl<256, 4>(p, grid, stream, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace moe
