// Decode path (1 <= T <= 8 tokens) as ONE persistent launch.
//
// At these sizes the layer streams weights (NemotronMoeLayer `decode`;
// MoeLayer `forward_k2` / `forward_k3` run a few tokens through one weight
// sweep): about 160 MB at T = 1 against a few MFLOP.  The pass runs as one
// cooperative grid of one CTA per SM.
//
// The work is cut along the experts' intermediate dimension.  A unit is 128
// intermediate rows of a routed slot's expert (64 for its last tile when the
// expert's size is an odd multiple of 64), or 64 rows of the shared expert:
//   up     u = relu^2(W_up[rows] . n) (x routing weight), 128 x 16 tokens,
//          K = H: tcgen05.mma M = 128 (weight rows; a 64-row unit loads
//          64-row boxes and leaves the other accumulator rows unused),
//          N = 16 (tokens), BF16 in, fp32 accumulate in TMEM;
//   down   y += W_down[:, rows] . u over all H output rows (K = 128 or 64), the
//          relu^2 rows going from TMEM through shared memory as the MMA's
//          token operand.
// A unit needs nothing from other CTAs once the tokens are routed, and every
// unit's down adds into the same H x 16 accumulator, which stays in TMEM
// (ceil(H / 128) x 16 columns) until the CTA's last unit.  Unit j goes to
// CTA j % grid: shared-expert units first (they need no routing and start at
// once), routed units after.  At the end every CTA adds its partial H x T
// block into an int64 fixed-point accumulator (integer addition: exact and
// independent of the order, so the result is deterministic), and each CTA
// finishes one slice of rows, the sum plus the residual, into hidden.
//
// Warp roles (320 threads):
//   warp 0     TMA producer: weight boxes (and the up GEMM's token rows) into
//              a ring of stages; up and down boxes interleave so a unit's
//              relu^2 rows are ready by the time its down boxes are consumed.
//   warp 1     TMEM owner and MMA issuer.
//   warps 2-5  epilogue: relu^2 rows into shared memory; the partial output.
//   warps 6-9  routing: one pass over this CTA's gate row(s) and the tokens
//              gives the sums of squares and the dot products at once,
//              logit = rsqrt(mean x^2 + eps) * (G_e . (x * w)) in fp32, and
//              the CTA's own copy of the bf16 normed rows (the up GEMM's token
//              operand); CTA 0 writes the residual.  Once every CTA's logits
//              are in, each CTA runs the same sigmoid top-k and builds the
//              same table of routed slots (distinct experts, first-use order).
//              With FP8 routed units they then dequantise the weight boxes
//              (or, W8A8 at one token, write an E4M3 copy of the token row).
//   all        the final reduction.
//
// Every wait is bounded (about one second): a timeout sets a status bit, the
// CTA drains its own TMA loads and MMAs, frees its TMEM and returns.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "decode.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {
namespace {

using bf16 = __nv_bfloat16;

// A stage holds kKB consecutive 64-wide k-blocks: kKB weight boxes, then
// (up only) kKB token boxes.  One TMA-completion barrier per two boxes
// streams about a third faster per SM than one per box at the same bytes in
// flight (measured with a standalone streaming probe on B200: 59 against
// 46 GB/s per SM with 90 SMs streaming).
constexpr int kKB = 2;
// Rows of a shared-expert unit.  Half the routed units' 128: twice as many
// CTAs stream the shared expert while the routing runs (its weights need no
// routing), 58 instead of 29 at shared_inter 3712.
constexpr int kSharedUnit = 64;
// W8A8 at one token (FusedParams::w8): the token chooses top_k distinct
// experts, and when their routed units fit on the CTAs beside the shared
// expert's, every such CTA has one unit, whose accumulators hold one
// expert's products alone.  The MMA then reads the E4M3 weight boxes from
// the staging slots as they land (kind::f8f6f4), with the token row and the
// relu^2 rows in E4M3 (one scale each, amax / 448), and the epilogues apply
// the weight row scales and those two scales: no dequantisation at all.
constexpr int kStages = 5;
constexpr int kABytes = kBM * 128;          // 128 weight rows x 64 BF16
constexpr int kBBytes = kDecodeN * 128;     // 16 token rows x 64 BF16
constexpr int kStageBytes = kKB * (kABytes + kBBytes);
// FP8 routed experts (E4M3 weights, one fp32 scale per weight row): the
// weights stream as FP8 boxes of 128 rows x 128 bytes (= one stage's two
// 64-wide k-blocks) into kF8Slots staging slots, with the up GEMM's token
// boxes beside them; the routing warps, idle once the routing is done,
// dequantise each box (value x its row's scale, rounded to BF16) into a BF16
// stage that the MMA reads as before.  Those CTAs keep kStagesF8 BF16
// stages.  The CTAs of the (BF16) shared expert use the same memory as
// kStages BF16 stages.
constexpr int kStagesF8 = 2;
constexpr int kF8Slots = 6;
constexpr int kF8ABytes = kBM * 128;              // 128 rows x 128 E4M3
constexpr int kF8SlotBytes = kF8ABytes + kKB * kBBytes;
constexpr int kRingBytesF8 = kStagesF8 * kStageBytes + kF8Slots * kF8SlotBytes;
constexpr int kRingBytes(bool f8) {
  return f8 && kRingBytesF8 > kStages * kStageBytes ? kRingBytesF8 : kStages * kStageBytes;
}
constexpr int kUBytes = 2 * kBBytes;        // a unit's relu^2 rows: 16 tokens x 128 K, two 64-wide chunks
constexpr int kThreads = 320;               // see the warp roles above
constexpr int kEpiThreads = 128;
constexpr int kRouteThreads = 128;
constexpr int kMaxSlots = kDecodeMaxT * kTopKMax;  // routed slots (distinct experts)
constexpr int kMaxChunks = 4;               // 8-element chunks per routing thread (H <= 4096)
constexpr int kTmemCols = 512;              // 2 x 16 (up) + ceil(H / 128) x 16 (down)
constexpr int kMaxRowTiles = kTmemCols / kDecodeN - 2;
constexpr int kSmemOf(bool f8) { return kRingBytes(f8) + 2 * kUBytes + 1024 + 1024; }

// Output rows that each CTA finishes: ceil(H / grid), rounded up to a
// multiple of 4 (vector loads and stores).
__host__ __device__ constexpr int reduce_rows(int H, int G) { return ((H + G - 1) / G + 3) & ~3; }

// The CTAs' partial outputs add up in a fixed-point accumulator: partial x
// is added as round(x * 2^24) to an int64, so the sum is exact and does not
// depend on the order in which the CTAs finish (every replay gives the same
// bits).  The rounding costs at most 2^-25 per partial, far below the bf16
// rounding of the result.  A partial that is NaN, infinite or larger than
// 2^31 in magnitude (where 148 of them could overflow the int64) marks its
// output element, which then comes out NaN.
constexpr float kFixScale = 16777216.0f;   // 2^24
constexpr float kFixLimit = 2147483648.0f;  // 2^31

// Named barriers (0 is __syncthreads).
constexpr int kBarEpi = 1;
constexpr int kBarRoute = 2;

// Synchronisation words of the workspace (FusedWorkspace::sync).
enum { kRouteArrived = 0, kPartialsDone = 1, kExited = 2 };

struct FusedParams {
  CUtensorMap tm_up;     // routed up weights   [E*I, H]  (A, 128-row boxes)
  CUtensorMap tm_sup;    // shared up weights   [S, H]
  CUtensorMap tm_down;   // routed down weights [E*H, I]
  CUtensorMap tm_sdown;  // shared down weights [H, S]
  CUtensorMap tm_up64;   // routed up weights, 64-row boxes (an expert's last 64-row tile)
  CUtensorMap tm_sup64;  // shared up weights, 64-row boxes (shared units are 64 rows)
  CUtensorMap tm_x8;     // x8 [grid * 16, H] E4M3 token rows (W8A8 launch), one-row boxes
  CUtensorMap tm_x;      // x16 [grid * 16, H]: 16 rows per CTA   (B, boxes of MAXT rows)
  const bf16* hidden;
  bf16* residual;
  bf16* out;             // hidden (in place) or another buffer; written at the very end
  const bf16* norm_w;
  const bf16* gate_w;
  const float* gate_bias;
  int w8;  // FP8 experts at one token, at most one routed unit per CTA: W8A8 (the note at kSharedUnit)
  const float* up_scale;    // [E, I] FP8 routed experts' row scales (else null)
  const float* down_scale;  // [E, H]
  int T, H, E, k, I, S;
  float eps, rsf;
  FusedWorkspace ws;
  int* status;
};

// ------------------------------------------------- memory-model helpers
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Release increment: this thread's earlier writes, and those of the threads
// it synchronised with through a barrier, become visible before the count.
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Order this thread's generic-proxy global accesses with its later
// async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Make this thread's shared-memory writes visible to the tensor cores.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void record_timeout(int* status, volatile int* abort) {
  *abort = 1;
  if (status) atomicOr(status, kStatusWaitTimeout);
}

// Bounded wait until *p >= target (acquire), polling every ~100 ns.  False
// on timeout or abort.
__device__ __forceinline__ bool wait_counter(const unsigned* p, unsigned target,
                                             volatile int* abort) {
  if (ld_acquire(p) >= target) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(100);
    if (ld_acquire(p) >= target) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
}

__device__ __forceinline__ float lo16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  f[0] = lo16(u.x); f[1] = hi16(u.x);
  f[2] = lo16(u.y); f[3] = hi16(u.y);
  f[4] = lo16(u.z); f[5] = hi16(u.z);
  f[6] = lo16(u.w); f[7] = hi16(u.w);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Eight floats as E4M3 (round to nearest even, saturating), in order.
__device__ __forceinline__ uint2 e4m3x8(const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int h = 0; h < 4; ++h)
    w[h] = __nv_cvt_float2_to_fp8x2(make_float2(v[2 * h], v[2 * h + 1]), __NV_SATFINITE, __NV_E4M3);
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// Shared state of one CTA.
struct Shared {
  uint64_t full[kStages], empty[kStages];
  uint64_t f8full[kF8Slots], f8empty[kF8Slots];  // FP8 staging slots: TMA -> dequantisation (or MMA, W8A8)
  uint64_t tfull[2], tempty[2];   // up accumulators: MMA -> epilogue -> MMA
  uint64_t ufull[2], ufree[2];    // relu^2 row buffers: epilogue -> MMA -> epilogue
  uint64_t down_done;             // every down MMA of the CTA has completed
  uint64_t loads_out;             // the routing warps' loads have returned
  uint64_t tokens;                // this CTA's normed rows are written (TMA may load them)
  uint64_t routed;                // the routing warps have built the slot table
  uint64_t warm;                  // the epilogue warps' dry routing pass is over
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int stop;                 // the epilogue warps' common decision to stop (epi_stop)
  int route_fail;
  int has_partial;          // the epilogue warps staged this CTA's partial output
  uint32_t partial_tokens;  // its token columns that are not exactly zero
  int flag;
  int U;                    // routed slots
  float rs[kDecodeMaxT];
  float red[4][kDecodeMaxT * 3];
  float amax8[4];           // W8A8: per-warp maxima (token row, then relu^2 rows)
  float x8s, u8s;           // W8A8: the E4M3 scales of the token row and of the relu^2 rows
  int seg_expert[kMaxSlots];            // expert of routed slot s
  float seg_w[kMaxSlots][kDecodeN];     // routing weight of token t in slot s (0 = not routed)
  int sel_idx[kDecodeMaxT * kTopKMax];
  float sel_w[kDecodeMaxT * kTopKMax];
  int first_use[kDecodeMaxT * kTopKMax];
  int slot_of[MOE_MAX_EXPERTS];
  float bias[MOE_MAX_EXPERTS];
};

static_assert(kSmemOf(false) + sizeof(Shared) <= 227 * 1024, "shared memory of one CTA");
static_assert(kDecodeMaxT * kMaxChunks * kRouteThreads * 8 * 4 <= kStages * kStageBytes,
              "a CTA's partial output [T, H] fp32 is staged in the idle ring");
static_assert(kSmemOf(true) + sizeof(Shared) <= 227 * 1024, "shared memory of one CTA (FP8)");
static_assert(kStagesF8 <= kStages, "barrier arrays");

// The four epilogue warps meet here and take one decision together:
// whether to stop (some role recorded a timeout).  Control flow of the
// epilogue warps never diverges, so their named barriers always complete.
__device__ __forceinline__ bool epi_stop(Shared& sh, int tid) {
  named_barrier(kBarEpi, kEpiThreads);
  if (tid == 0) sh.stop = sh.abort;
  named_barrier(kBarEpi, kEpiThreads);
  return sh.stop != 0;
}

// ------------------------------------------------------------------ units
// Units: shared-expert tiles j < nS, then routed tile (j - nS) % nI of slot
// (j - nS) / nI.  CTA c takes j = c, c + grid, c + 2 grid, ...  (Neighbouring
// CTAs thus stream neighbouring tiles of an expert at the same time; its
// down slices share DRAM rows.  Giving each CTA a contiguous run of routed
// tiles instead made the T = 8 stream about 8 us slower.)  With FP8
// routed experts the two kinds stay on separate CTAs (a CTA's stages are
// either BF16 or FP8): CTA c < nS takes shared unit c alone, and the routed
// units go round-robin over the other Gr = grid - nS CTAs.  Its steps:
// the up of each unit and the down of each unit, ordered so that a unit's
// down comes one unit after its up (the relu^2 rows are ready by then),
// except that a shared first unit is followed by its own down at once (its
// successors wait for the routing).
struct Units {
  int c, G, nS, nI, N;  // N = nS + U * nI, the units of the pass (known after routing)
  bool f8;              // FP8 routed experts: shared and routed units on separate CTAs
  __device__ __forceinline__ int count() const {
    if (!f8) return c < N ? (N - 1 - c) / G + 1 : 0;
    if (c < nS) return 1;
    const int r = c - nS, nr = N - nS, Gr = G - nS;
    return r < nr ? (nr - 1 - r) / Gr + 1 : 0;
  }
  __device__ __forceinline__ int unit(int n) const {
    if (!f8) return c + n * G;
    return c < nS ? c : c + n * (G - nS);
  }
  __device__ __forceinline__ bool shared_first() const { return c < nS; }
};

// The s-th step of a CTA with m units: kind 0 = up, 1 = down, of its unit n.
// m = 0 (routing not yet known) gives the steps that do not depend on it:
// with a shared first unit, its up and its down.
__device__ __forceinline__ bool step_of(const Units& u, int m, int s, int* kind, int* n) {
  if (u.shared_first()) {
    if (s == 0) { *kind = 0; *n = 0; return true; }
    if (s == 1) { *kind = 1; *n = 0; return true; }
    s -= 2;
    // routed units 1 .. m-1: up(1), up(2), down(1), up(3), down(2), ..., down(m-1)
    const int r = m - 1;
    if (r <= 0) return false;
    if (s == 0) { *kind = 0; *n = 1; return true; }
    // after the first up: pairs (up(i + 1), down(i)) for i = 1 .. r - 1, then down(r)
    const int q = s - 1;
    const int i = 1 + q / 2;
    if (i < r) {
      *kind = (q & 1) ? 1 : 0;
      *n = (q & 1) ? i : i + 1;
      return true;
    }
    if (q == 2 * (r - 1)) { *kind = 1; *n = r; return true; }
    return false;
  }
  // up(0), up(1), down(0), up(2), down(1), ..., down(m-1)
  if (m <= 0) return false;
  if (s == 0) { *kind = 0; *n = 0; return true; }
  const int q = s - 1;
  const int i = q / 2;
  if (i < m - 1) {
    *kind = (q & 1) ? 1 : 0;
    *n = (q & 1) ? i : i + 1;
    return true;
  }
  if (q == 2 * (m - 1)) { *kind = 1; *n = m - 1; return true; }
  return false;
}

// ---------------------------------------------------------------- routing
// Routing warps (rt 0..127).  One pass over the tokens, the norm weight and
// this CTA's gate rows (blockIdx.x and, with E > grid, blockIdx.x + grid)
// gives everything at once: the sums of squares, the dot products
// G_e . (x_t * w), this CTA's copy of the token rows bf16(x * w) for the up
// GEMM, and (CTA 0) the residual.  The up GEMM's token operand leaves out
// the factor r_t = rsqrt(mean x_t^2 + eps), so it needs nothing but the
// loads; the epilogue applies r_t to accumulator column t instead
// (W . (x r w) = r (W . (x w))).
//
// One or two tokens: every routing thread takes chunks rt, rt + 128, ...
// of every token, and all their loads are in flight at once, issued first
// of all, before the launch's set-up (route_issue): the routing decides
// when the routed weights can stream, and the set-up's cold instruction
// fetches then overlap the loads' DRAM latency (2.5 us earlier routing at
// T = 1).
//
// Three or four tokens: the same mapping, two chunks' loads in flight at a
// time.  Five to eight tokens: routing warp w owns tokens w and w + 4, and
// its lanes stride over the chunks, kTokChunks of them in flight
// (route_tokwarp).  Unrolled over eight tokens, the first mapping's loop
// body is large, and its first pass (cold instruction cache after the L2
// flush) took about 3.5 us per chunk; the token rows are then ready 2.8 us
// later at T = 8 (at T = 4 the warp-per-token loop, with three rounds of
// loads instead of two, is 0.5 us slower).
template <int MAXT>
struct RouteLoads {
  static constexpr bool kHold = MAXT <= 2;
  static constexpr bool kTokWarp = MAXT > 4;
  static constexpr int kHeld = kHold ? kMaxChunks : 2;  // (3-4 tokens: two chunks at a time)
  uint4 x[kHeld][MAXT], w[kHeld], a[kHeld], b[kHeld];
};
constexpr int kTokChunks = 4;  // chunks in flight per lane with a warp per token

// Chunk j of routing thread rt: the norm weight, this CTA's gate rows and
// the tokens, 8 elements each.
template <int MAXT>
__device__ __forceinline__ void route_load_chunk(const FusedParams& p, int rt, int j,
                                                 uint4 (&x)[MAXT], uint4& w, uint4& a, uint4& b) {
  const int H = p.H, E = p.E, G = gridDim.x;
  const int e0 = blockIdx.x, e1 = blockIdx.x + G;
  const int c = rt + j * kRouteThreads;
  const bool in = c < H / 8;
  w = in ? __ldg(reinterpret_cast<const uint4*>(p.norm_w) + c) : make_uint4(0, 0, 0, 0);
  a = in && e0 < E ? __ldcs(reinterpret_cast<const uint4*>(p.gate_w + size_t(e0) * H) + c)
                   : make_uint4(0, 0, 0, 0);
  b = in && e1 < E ? __ldcs(reinterpret_cast<const uint4*>(p.gate_w + size_t(e1) * H) + c)
                   : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int t = 0; t < MAXT; ++t)
    x[t] = in && t < p.T ? reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[c]
                         : make_uint4(0, 0, 0, 0);
}

template <int MAXT>
__device__ __forceinline__ void route_issue(const FusedParams& p, int rt, RouteLoads<MAXT>& L) {
  if constexpr (RouteLoads<MAXT>::kHold) {
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j)
      route_load_chunk<MAXT>(p, rt, j, L.x[j], L.w[j], L.a[j], L.b[j]);
  }
}

// Five to eight tokens (see RouteLoads): warp w of the routing warps sums
// tokens w and w + 4 over all of H, lane l taking chunks l, l + 32, ...,
// kTokChunks at a time.  The norm weight and this CTA's gate rows are loaded
// by every warp (L2 hits after the first).  Same products as route_hold;
// each token's sums are reduced within its warp.
template <int MAXT>
__device__ __forceinline__ void route_tokwarp(const FusedParams& p, Shared& sh, int rt,
                                              bool f16tok) {
  constexpr int TPW = (MAXT + 3) / 4;  // tokens per warp
  const int H = p.H, T = p.T, E = p.E, G = gridDim.x;
  const int nv = H / 8;
  const int warp = rt >> 5, lane = rt & 31;
  const int e0 = blockIdx.x, e1 = blockIdx.x + G;
  const bool has0 = e0 < E, has1 = e1 < E;
  bf16* x16 = p.ws.x16 + size_t(blockIdx.x) * kDecodeN * H;
  float ss[TPW], d0[TPW], d1[TPW];
#pragma unroll
  for (int i = 0; i < TPW; ++i) ss[i] = d0[i] = d1[i] = 0.f;
  if (warp < T) {
#pragma unroll 1
    for (int c0 = lane; c0 < nv; c0 += 32 * kTokChunks) {
      uint4 xq[kTokChunks][TPW], wq[kTokChunks], aq[kTokChunks], bq[kTokChunks];
#pragma unroll
      for (int u = 0; u < kTokChunks; ++u) {
        const int c = c0 + 32 * u;
        const bool in = c < nv;
        const uint4 z = make_uint4(0, 0, 0, 0);
        wq[u] = in ? __ldg(reinterpret_cast<const uint4*>(p.norm_w) + c) : z;
        aq[u] = in && has0 ? __ldcs(reinterpret_cast<const uint4*>(p.gate_w + size_t(e0) * H) + c)
                           : z;
        bq[u] = in && has1 ? __ldcs(reinterpret_cast<const uint4*>(p.gate_w + size_t(e1) * H) + c)
                           : z;
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const int t = warp + 4 * i;
          xq[u][i] = in && t < T ? reinterpret_cast<const uint4*>(p.hidden + size_t(t) * H)[c] : z;
        }
      }
#pragma unroll
      for (int u = 0; u < kTokChunks; ++u) {
        const int c = c0 + 32 * u;
        float w[8], a[8], b[8];
        unpack8(wq[u], w);
        unpack8(aq[u], a);
        unpack8(bq[u], b);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          a[q] *= w[q];
          b[q] *= w[q];
        }
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const int t = warp + 4 * i;
          float f[8];
          unpack8(xq[u][i], f);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            ss[i] += f[q] * f[q];
            d0[i] += a[q] * f[q];
            d1[i] += b[q] * f[q];
          }
          if (c < nv && t < T) {
            reinterpret_cast<uint4*>(x16 + size_t(t) * H)[c] =
                f16tok ? make_uint4(pack_f16x2(f[0] * w[0], f[1] * w[1]),
                                    pack_f16x2(f[2] * w[2], f[3] * w[3]),
                                    pack_f16x2(f[4] * w[4], f[5] * w[5]),
                                    pack_f16x2(f[6] * w[6], f[7] * w[7]))
                       : make_uint4(pack_bf16x2(f[0] * w[0], f[1] * w[1]),
                                    pack_bf16x2(f[2] * w[2], f[3] * w[3]),
                                    pack_bf16x2(f[4] * w[4], f[5] * w[5]),
                                    pack_bf16x2(f[6] * w[6], f[7] * w[7]));
            if (blockIdx.x == 0) reinterpret_cast<uint4*>(p.residual + size_t(t) * H)[c] = xq[u][i];
          }
        }
      }
    }
  }
  if (rt < E) sh.bias[rt] = p.gate_bias ? p.gate_bias[rt] : 0.f;
  if (rt + kRouteThreads < E)
    sh.bias[rt + kRouteThreads] = p.gate_bias ? p.gate_bias[rt + kRouteThreads] : 0.f;
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    const int t = warp + 4 * i;
    const float v0 = warp_sum(ss[i]), v1 = warp_sum(d0[i]), v2 = warp_sum(d1[i]);
    if (lane == 0 && t < T) {
      const float r = rsqrtf(v0 / float(H) + p.eps);
      sh.rs[t] = r;
      if (has0) p.ws.logits[t * E + e0] = v1 * r;
      if (has1) p.ws.logits[t * E + e1] = v2 * r;
    }
  }
  // the token rows: generic writes -> the TMA loads of this CTA's producer
  fence_proxy_async_global();
  named_barrier(kBarRoute, kRouteThreads);
  // the token rows, their factors r_t and every logit of this CTA are in
  // place (and, CTA 0, the residual): the weight stream may start
  if (rt == 0) {
    mbar_arrive(&sh.loads_out);
    mbar_arrive(&sh.tokens);
    red_release_add(p.ws.sync + kRouteArrived, 1u);
  }
}

// One to four tokens (see RouteLoads); with one or two, from the loads
// route_issue made.  F8: the launch has FP8 routed experts (only then may
// it write the E4M3 token row of W8A8).
template <int MAXT, bool F8>
__device__ void route_hold(const FusedParams& p, Shared& sh, int rt, RouteLoads<MAXT>& L,
                           bool f16tok) {
  const int H = p.H, T = p.T, E = p.E, G = gridDim.x;
  const int nv = H / 8;
  const int warp = rt >> 5, lane = rt & 31;
  const int e0 = blockIdx.x, e1 = blockIdx.x + G;
  const bool has0 = e0 < E, has1 = e1 < E;
  bf16* x16 = p.ws.x16 + size_t(blockIdx.x) * kDecodeN * H;
  float ss[MAXT], d0[MAXT], d1[MAXT];
#pragma unroll
  for (int t = 0; t < MAXT; ++t) ss[t] = d0[t] = d1[t] = 0.f;
  // sums of chunk j, and its token rows bf16(x * w) (and the residual)
  auto consume = [&](int j, const uint4 (&x)[MAXT], const uint4& wq, const uint4& aq,
                     const uint4& bq) {
    const int c = rt + j * kRouteThreads;
    float w[8], a[8], b[8];
    unpack8(wq, w);
    unpack8(aq, a);
    unpack8(bq, b);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      a[q] *= w[q];
      b[q] *= w[q];
    }
#pragma unroll
    for (int t = 0; t < MAXT; ++t) {
      float f[8];
      unpack8(x[t], f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        ss[t] += f[q] * f[q];
        d0[t] += a[q] * f[q];
        d1[t] += b[q] * f[q];
      }
      if (c < nv && t < T) {
        reinterpret_cast<uint4*>(x16 + size_t(t) * H)[c] =
            f16tok ? make_uint4(pack_f16x2(f[0] * w[0], f[1] * w[1]),
                                pack_f16x2(f[2] * w[2], f[3] * w[3]),
                                pack_f16x2(f[4] * w[4], f[5] * w[5]),
                                pack_f16x2(f[6] * w[6], f[7] * w[7]))
                   : make_uint4(pack_bf16x2(f[0] * w[0], f[1] * w[1]),
                                pack_bf16x2(f[2] * w[2], f[3] * w[3]),
                                pack_bf16x2(f[4] * w[4], f[5] * w[5]),
                                pack_bf16x2(f[6] * w[6], f[7] * w[7]));
        if (blockIdx.x == 0) reinterpret_cast<uint4*>(p.residual + size_t(t) * H)[c] = x[t];
      }
    }
  };
  if constexpr (RouteLoads<MAXT>::kHold) {
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j) consume(j, L.x[j], L.w[j], L.a[j], L.b[j]);
  } else {
    // two chunks' loads in flight at a time
#pragma unroll 1
    for (int j = 0; j < kMaxChunks; j += 2) {
      route_load_chunk<MAXT>(p, rt, j, L.x[0], L.w[0], L.a[0], L.b[0]);
      route_load_chunk<MAXT>(p, rt, j + 1, L.x[1], L.w[1], L.a[1], L.b[1]);
      consume(j, L.x[0], L.w[0], L.a[0], L.b[0]);
      consume(j + 1, L.x[1], L.w[1], L.a[1], L.b[1]);
    }
  }
  if (rt < E) sh.bias[rt] = p.gate_bias ? p.gate_bias[rt] : 0.f;
  if (rt + kRouteThreads < E)
    sh.bias[rt + kRouteThreads] = p.gate_bias ? p.gate_bias[rt + kRouteThreads] : 0.f;
#pragma unroll
  for (int t = 0; t < MAXT; ++t) {
    const float v0 = warp_sum(ss[t]), v1 = warp_sum(d0[t]), v2 = warp_sum(d1[t]);
    if (lane == 0) {
      sh.red[warp][t] = v0;
      sh.red[warp][MAXT + t] = v1;
      sh.red[warp][2 * MAXT + t] = v2;
    }
  }
  // W8A8 (one token, FP8 units): the E4M3 copy of x * w needs the row's
  // maximum |x * w| first
  const bool want8 = F8 && f16tok && p.w8;
  if constexpr (F8 && RouteLoads<MAXT>::kHold) if (want8) {
    float xm = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j) {
      float f[8], g[8];
      unpack8(L.x[j][0], f);
      unpack8(L.w[j], g);
#pragma unroll
      for (int q = 0; q < 8; ++q) xm = fmaxf(xm, fabsf(f[q] * g[q]));  // (zeros past H)
    }
    xm = warp_max(xm);
    if (lane == 0) sh.amax8[warp] = xm;
  }
  // the token rows: generic writes -> the TMA loads of this CTA's producer
  fence_proxy_async_global();
  named_barrier(kBarRoute, kRouteThreads);
  // the routing loads have returned (their sums are in shared memory): the
  // weight stream may start.  Routing decides when the routed weights can
  // stream, so its loads go first.
  if (rt == 0) mbar_arrive(&sh.loads_out);
  if constexpr (F8 && RouteLoads<MAXT>::kHold) if (want8) {
    const float mx = fmaxf(fmaxf(sh.amax8[0], sh.amax8[1]), fmaxf(sh.amax8[2], sh.amax8[3]));
    const float s8 = mx > 0.f ? mx / 448.f : 1.f;
    const float inv = 1.f / s8;
    if (rt == 0) sh.x8s = s8;
    uint2* x8 = reinterpret_cast<uint2*>(p.ws.x8 + size_t(blockIdx.x) * kDecodeN * H);
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j) {
      const int c = rt + j * kRouteThreads;
      if (c < nv) {
        float f[8], g[8];
        unpack8(L.x[j][0], f);
        unpack8(L.w[j], g);
#pragma unroll
        for (int q = 0; q < 8; ++q) f[q] = f[q] * g[q] * inv;
        x8[c] = e4m3x8(f);
      }
    }
    fence_proxy_async_global();  // (the E4M3 row -> this CTA's TMA loads)
  }
  if (rt < T) {
    float s = 0.f, a = 0.f, b = 0.f;
    for (int w = 0; w < 4; ++w) {
      s += sh.red[w][rt];
      a += sh.red[w][MAXT + rt];
      b += sh.red[w][2 * MAXT + rt];
    }
    const float r = rsqrtf(s / float(H) + p.eps);
    sh.rs[rt] = r;
    if (has0) p.ws.logits[rt * E + e0] = a * r;
    if (has1) p.ws.logits[rt * E + e1] = b * r;
  }
  named_barrier(kBarRoute, kRouteThreads);
  // the token rows and their factors r_t are in place; every logit of this
  // CTA is written (and, CTA 0, the residual)
  if (rt == 0) {
    mbar_arrive(&sh.tokens);
    red_release_add(p.ws.sync + kRouteArrived, 1u);
  }
}

// The routing pass of the routing warps (see RouteLoads).  f16tok: write the
// token rows as f16 instead of BF16 (the up GEMM of FP8 units runs on f16
// operands).
template <int MAXT, bool F8>
__device__ __forceinline__ void route_logits(const FusedParams& p, Shared& sh, int rt,
                                             RouteLoads<MAXT>& L, bool f16tok) {
  if constexpr (RouteLoads<MAXT>::kTokWarp)
    route_tokwarp<MAXT>(p, sh, rt, f16tok);
  else
    route_hold<MAXT, F8>(p, sh, rt, L, f16tok);
}

// The sigmoid top-k of token t by one warp, into sel_idx / sel_w.  The dry
// pass (see route_select) loads no logits: it must only run the same
// instructions, and a load from DRAM would hold it up.
__device__ __forceinline__ void topk_of_token(const FusedParams& p, Shared& sh, int t, int lane,
                                              bool dry) {
  const int E = p.E;
  float lg[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    lg[j] = !dry && lane + 32 * j < E ? __ldcg(p.ws.logits + t * E + lane + 32 * j) : 0.f;
  warp_topk_regs(lg, p.gate_bias ? sh.bias : nullptr, E, p.k, p.rsf, sh.sel_idx + t * p.k,
                 sh.sel_w + t * p.k);
}

// Once every CTA's logits are in: the sigmoid top-k of every token and the
// routed slot table (identical in every CTA).  Returns false on timeout.
//
// The same code also runs once as a dry pass, by the epilogue warps at the
// start of the launch (barrier `bar`, dry = true): it reads whatever the
// logits buffer holds, writes only the CTA's own tables (which the real pass
// rewrites whole) and nothing global.  Its point is the instruction cache:
// the real pass sits on the critical path of every routed unit, and after
// the working set has left L2 its first run would otherwise fetch each
// instruction line from DRAM.  Not inlined, so that both passes run the same
// instructions.
__device__ __noinline__ bool route_select(const FusedParams& p, Shared& sh, int rt,
                                          volatile int* abort, int bar, bool dry) {
  const int T = p.T, E = p.E, k = p.k;
  const int warp = rt >> 5, lane = rt & 31;
  if (!dry) {
    if (rt == 0) {
      sh.route_fail = 0;
      // the dry pass has left the tables, and every CTA's logits are in
      if (!mbar_wait(&sh.warm, 0, abort) ||
          !wait_counter(p.ws.sync + kRouteArrived, gridDim.x, abort)) {
        record_timeout(p.status, abort);
        sh.route_fail = 1;
      }
    }
    named_barrier(bar, kRouteThreads);
    if (sh.route_fail) return false;
  }
  if (T == 1) {
    // One token: its k choices are distinct experts, and slot s is choice s.
    // One warp does it all (no table scan, no further barriers but the last).
    if (warp == 0) {
      topk_of_token(p, sh, 0, lane, dry);
      for (int i = lane; i < k * kDecodeN; i += 32) (&sh.seg_w[0][0])[i] = 0.f;
      __syncwarp();
      if (lane < k) {
        const int e = sh.sel_idx[lane];
        const float w = sh.sel_w[lane];
        if (!dry && blockIdx.x == 0) {  // the routing of the pass, for moe_copy_routing
          p.ws.idx[lane] = e;
          p.ws.w[lane] = w;
        }
        // an id outside [0, E) (only from NaN logits) is routed nowhere
        const bool valid = unsigned(e) < unsigned(E);
        sh.seg_expert[lane] = valid ? e : 0;
        if (valid) sh.seg_w[lane][0] = w;
        if (!valid && !dry) atomicOr(p.status, kStatusBadIndex);
      }
      if (lane == 0) sh.U = k;
    }
    named_barrier(bar, kRouteThreads);
    return true;
  }
  for (int t = warp; t < T; t += 4) topk_of_token(p, sh, t, lane, dry);
  for (int i = rt; i < kMaxSlots * kDecodeN; i += kRouteThreads) (&sh.seg_w[0][0])[i] = 0.f;
  named_barrier(bar, kRouteThreads);
  const int R = T * k;
  for (int f = rt; f < R; f += kRouteThreads) {
    const int e = sh.sel_idx[f];
    int first = 1;
    for (int g = 0; g < f; ++g) first &= sh.sel_idx[g] != e;
    sh.first_use[f] = first;
    if (!dry && blockIdx.x == 0) {  // the routing of the pass, for moe_copy_routing
      p.ws.idx[f] = e;
      p.ws.w[f] = sh.sel_w[f];
    }
  }
  named_barrier(bar, kRouteThreads);
  if (warp == 0) {  // exclusive scan of the first-use flags (R <= 128)
    int base = 0;
    for (int f0 = 0; f0 < R; f0 += 32) {
      const int f = f0 + lane;
      const int v = f < R ? sh.first_use[f] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (v) {
        const int e = sh.sel_idx[f];
        if (unsigned(e) < unsigned(E)) sh.slot_of[e] = base + incl - 1;
        sh.seg_expert[base + incl - 1] = e;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) sh.U = base;
  }
  named_barrier(bar, kRouteThreads);
  for (int f = rt; f < R; f += kRouteThreads) {
    const int e = sh.sel_idx[f];
    if (unsigned(e) < unsigned(E)) sh.seg_w[sh.slot_of[e]][f / k] = sh.sel_w[f];
  }
  // an id outside [0, E) (only from NaN logits) is routed nowhere
  for (int s = rt; s < sh.U; s += kRouteThreads)
    if (unsigned(sh.seg_expert[s]) >= unsigned(E)) {
      sh.seg_expert[s] = 0;
      if (!dry) atomicOr(p.status, kStatusBadIndex);
    }
  named_barrier(bar, kRouteThreads);
  return true;
}


// ------------------------------------------------------------- epilogue
// The relu^2 rows of a unit go into a shared-memory buffer laid out exactly
// as a TMA box of the token operand would be (16 token rows x 64 K per 2 KB
// chunk, 128-byte swizzle: the 16-byte chunk j of row t sits at j ^ (t % 8)),
// so the down MMA reads it with the usual descriptor.
__device__ __forceinline__ void store_u_row(uint8_t* ubuf, int rloc, const float (&v)[kDecodeN]) {
  const int kk = rloc >> 6, k = rloc & 63;
  uint8_t* base = ubuf + kk * kBBytes + (k & 7) * 2;
#pragma unroll
  for (int t = 0; t < kDecodeN; ++t)
    *reinterpret_cast<bf16*>(base + t * 128 + ((((k >> 3) ^ (t & 7)) & 7) << 4)) =
        __float2bfloat16_rn(v[t]);
}

// Unit n of CTA c: shared tile j < nS, or routed tile (j - nS) % nI of slot
// (j - nS) / nI.
struct UnitInfo {
  bool shared;
  int slot, expert, row0;
  int row_end;  // first intermediate row past the unit (64 or 128 rows after row0, or S / I)
};

__device__ __forceinline__ UnitInfo unit_info(const FusedParams& p, const Shared& sh,
                                              const Units& u, int n) {
  UnitInfo f;
  const int j = u.unit(n);
  f.shared = j < u.nS;
  if (f.shared) {
    f.slot = -1;
    f.expert = 0;
    f.row0 = j * kSharedUnit;
    f.row_end = min(p.S, f.row0 + kSharedUnit);
  } else {
    const int r = j - u.nS;
    f.slot = r / u.nI;
    f.expert = sh.seg_expert[f.slot];
    f.row0 = (r - f.slot * u.nI) * kBM;
    f.row_end = min(p.I, f.row0 + kBM);
  }
  return f;
}

// 64-wide k-blocks of a unit's down slice (64 or 128 rows: S and I are
// multiples of 64).
__device__ __forceinline__ int down_kk(const UnitInfo& f) { return f.row_end - f.row0 > 64 ? 2 : 1; }

// ------------------------------------------------------ FP8 dequantisation
// Row r of FP8 staging slot f8 (128 rows x 128 E4M3, 128-byte swizzle: the
// 16-byte chunk j of row r sits at j ^ (r % 8)) into BF16-layout stage st:
// its two 64-wide k-blocks, same swizzle, zeros for a row outside the
// matrix.
//   up:   f16, exactly the E4M3 values (every E4M3 value is an f16); the
//         row's scale is applied to the accumulator row in the epilogue, and
//         the tokens are f16 too.  The thread also copies its 32 bytes of
//         the two token boxes.
//   down: BF16 of the value times the row's scale (the product in f16,
//         rounded once more to BF16): the down accumulator adds units of
//         different experts, so each weight row carries its own scale.
template <bool UP>
__device__ __forceinline__ void dequant_row(const uint8_t* f8, uint8_t* st, int r, float scale,
                                            bool valid) {
  const uint8_t* src = f8 + r * 128;
  const __half2 s2 = __float2half2_rn(scale);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 q = *reinterpret_cast<const uint4*>(src + ((j ^ (r & 7)) << 4));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      __half2 lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[h] & 0xFFFFu),
                                              __NV_E4M3);
      __half2 hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[h] >> 16),
                                              __NV_E4M3);
      if constexpr (UP) {
        o[2 * h] = valid ? *reinterpret_cast<uint32_t*>(&lo) : 0u;
        o[2 * h + 1] = valid ? *reinterpret_cast<uint32_t*>(&hi) : 0u;
      } else {
        const float2 a = __half22float2(__hmul2(lo, s2)), b = __half22float2(__hmul2(hi, s2));
        o[2 * h] = valid ? pack_bf16x2(a.x, a.y) : 0u;
        o[2 * h + 1] = valid ? pack_bf16x2(b.x, b.y) : 0u;
      }
    }
    // E4M3 elements 16 j .. 16 j + 15 are chunks 2 (j % 4) and 2 (j % 4) + 1
    // of k-block j / 4
    uint8_t* dst = st + (j >> 2) * kABytes + r * 128;
    const int c0 = (j & 3) * 2;
    *reinterpret_cast<uint4*>(dst + ((c0 ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(dst + (((c0 + 1) ^ (r & 7)) << 4)) =
        make_uint4(o[4], o[5], o[6], o[7]);
  }
  if constexpr (UP) {
    const uint4* tb = reinterpret_cast<const uint4*>(f8 + kF8ABytes) + 2 * r;
    uint4* db = reinterpret_cast<uint4*>(st + kKB * kABytes) + 2 * r;
    db[0] = tb[0];
    db[1] = tb[1];
  }
}

// ------------------------------------------------------------ reduction
// Adds this CTA's partial value v of output element `at` (token-major
// [T, H]) into the fixed-point accumulator.
__device__ __forceinline__ void add_partial(const FusedWorkspace& ws, size_t at, float v) {
  if (fabsf(v) <= kFixLimit)  // (false for NaN)
    atomicAdd(reinterpret_cast<unsigned long long*>(ws.acc + at),
              static_cast<unsigned long long>(__float2ll_rn(v * kFixScale)));
  else
    ws.bad[at] = 1;
}

// Output rows [r0, r0 + nr) of T tokens, once every CTA has added its
// partial: the accumulated sum plus the input row, rounded once to bf16,
// into out; the accumulator and the marks of these elements are left at
// zero for the next launch.  Four rows per thread and step.
//
// Like route_select it also runs once as a dry pass at the start of the
// launch (epilogue warps, one token, four rows, no store), so that its
// instructions are in the cache when the real pass comes last on the
// critical path.  Not inlined, so that both passes run the same code.
__device__ __noinline__ void finish_slice(const FusedParams& p, int T, int r0, int nr, int tid,
                                          int nthreads, bool dry) {
  const int H = p.H;
  const int nq = nr >> 2;
  for (int i = tid; i < T * nq; i += nthreads) {
    const int t = i / nq;
    const size_t at = size_t(t) * H + r0 + (i - t * nq) * 4;
    const longlong2 q0 = __ldcg(reinterpret_cast<const longlong2*>(p.ws.acc + at));
    const longlong2 q1 = __ldcg(reinterpret_cast<const longlong2*>(p.ws.acc + at) + 1);
    const unsigned bad = __ldcg(reinterpret_cast<const unsigned*>(p.ws.bad + at));
    const uint2 hv = *reinterpret_cast<const uint2*>(p.hidden + at);
    const float m[4] = {float(q0.x) * (1.0f / kFixScale), float(q0.y) * (1.0f / kFixScale),
                        float(q1.x) * (1.0f / kFixScale), float(q1.y) * (1.0f / kFixScale)};
    const float x[4] = {lo16(hv.x), hi16(hv.x), lo16(hv.y), hi16(hv.y)};
    float o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = (bad >> (8 * j)) & 0xffu ? __int_as_float(0x7fc00000) : x[j] + m[j];
    if (!dry) {
      *reinterpret_cast<uint2*>(p.out + at) =
          make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
      reinterpret_cast<longlong2*>(p.ws.acc + at)[0] = make_longlong2(0, 0);
      reinterpret_cast<longlong2*>(p.ws.acc + at)[1] = make_longlong2(0, 0);
      if (bad) *reinterpret_cast<unsigned*>(p.ws.bad + at) = 0u;
    }
  }
}

// The routing warps' second job in a CTA with FP8 routed units: every stage
// of the CTA's steps, in the producer's and the MMA's order, from its FP8
// staging slot into the next BF16 stage (which the MMA frees), then the
// stage to the MMA and the slot back to the producer.  Returns false on a
// timeout (recorded).
__device__ bool dequant_stages(const FusedParams& p, Shared& sh, const Units& un, uint8_t* tiles,
                               int rt, volatile int* abort) {
  const int kbH = p.H / 64, nH = (p.H + kBM - 1) / kBM;
  uint8_t* slots = tiles + kStagesF8 * kStageBytes;
  int st = 0, fs = 0;
  uint32_t sph = 0, fph = 0;
  const int m = un.count();
  for (int s = 0;; ++s) {
    int kind, n;
    if (!step_of(un, m, s, &kind, &n)) break;
    const UnitInfo f = unit_info(p, sh, un, n);
    const int nstage = kind == 0 ? (kbH + kKB - 1) / kKB : nH;
    // down: this thread's row scales for the whole step (one per 128-row
    // block of the output, row i * 128 + rt), loaded before its first stage
    // (a scale load per stage would put a memory round trip into every
    // stage); up needs none here (the epilogue applies them)
    float sc[kMaxRowTiles];
#pragma unroll
    for (int i = 0; i < kMaxRowTiles; ++i) {
      const int row = i * kBM + rt;
      sc[i] = kind == 1 && i < nH && row < p.H ? p.down_scale[size_t(f.expert) * p.H + row]
                                               : 0.f;
    }
#pragma unroll 1
    for (int i = 0; i < nstage; ++i) {
      // Each warp on its own (no named barrier between the four): lane 0
      // waits (bounded) for the slot's data and the stage's room, the warp
      // takes its decision, converts its 32 rows and counts itself in on
      // the stage and the slot (four arrivals each).
      const int lane = rt & 31;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&sh.f8full[fs], fph, abort) && mbar_wait(&sh.empty[st], sph ^ 1u, abort);
        if (!ok) record_timeout(p.status, abort);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
      // (both phases are complete: every thread observes them itself)
      mbar_wait(&sh.f8full[fs], fph, abort);
      mbar_wait(&sh.empty[st], sph ^ 1u, abort);
      // up: weight row = intermediate row f.row0 + rt of the expert; down:
      // weight row = output row i * 128 + rt
      bool valid;
      float scale;
      if (kind == 0) {
        valid = f.row0 + rt < f.row_end;
        scale = 1.f;
      } else {
        valid = i * kBM + rt < p.H;
        scale = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxRowTiles; ++j)
          if (j == i) scale = sc[j];
      }
      if (kind == 0)
        dequant_row<true>(slots + fs * kF8SlotBytes, tiles + st * kStageBytes, rt, scale, valid);
      else
        dequant_row<false>(slots + fs * kF8SlotBytes, tiles + st * kStageBytes, rt, scale, valid);
      fence_proxy_async_shared();  // generic writes -> tensor core reads
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sh.full[st]);
        mbar_arrive(&sh.f8empty[fs]);
      }
      if (++st == kStagesF8) {
        st = 0;
        sph ^= 1u;
      }
      if (++fs == kF8Slots) {
        fs = 0;
        fph ^= 1u;
      }
    }
  }
  return true;
}

// ---------------------------------------------------------------- kernel
template <int MAXT, bool F8>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(const __grid_constant__ FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* tiles = smem_raw + pad;
  uint8_t* ubufs = tiles + kRingBytes(F8);  // two relu^2 row buffers
  Shared& sh = *reinterpret_cast<Shared*>(ubufs + 2 * kUBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool kStagePartial = MAXT >= 4;
  const int G = gridDim.x, cta = blockIdx.x;
  const int nH = (p.H + kBM - 1) / kBM;
  const int kbH = p.H / 64;

  Units un;
  un.c = cta;
  un.G = G;
  un.nS = (p.S + kSharedUnit - 1) / kSharedUnit;
  un.nI = (p.I + kBM - 1) / kBM;
  un.N = un.nS;  // the routed units are added once the routing is known
  un.f8 = F8;
  // this CTA's units are FP8 (dequantised by the routing warps, or read by the MMA under W8A8), and the
  // BF16 stages it has
  const bool conv = F8 && cta >= un.nS;
  const int nst = conv ? kStagesF8 : kStages;

  RouteLoads<MAXT> rl;
  if (warp >= 6) route_issue<MAXT>(p, threadIdx.x - 192, rl);

  if (threadIdx.x == 0) {
    // (a dequantising CTA's stages are filled by the four routing warps)
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], conv ? kRouteThreads / 32 : 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.tfull[b], 1);
      mbar_init(&sh.tempty[b], 4);
      mbar_init(&sh.ufull[b], 1);
      mbar_init(&sh.ufree[b], 1);
    }
    mbar_init(&sh.down_done, 1);
    mbar_init(&sh.loads_out, 1);
    mbar_init(&sh.tokens, 1);
    mbar_init(&sh.routed, 1);
    mbar_init(&sh.warm, 1);
    mbar_init(&sh.drain, 1);
    if (F8) {
      for (int s = 0; s < kF8Slots; ++s) {
        mbar_init(&sh.f8full[s], 1);
        // freed by the four dequantising warps, or under W8A8 by the MMA
        mbar_init(&sh.f8empty[s], p.w8 ? 1 : kRouteThreads / 32);
      }
    }
    sh.abort = 0;
    sh.U = 0;
    sh.has_partial = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_up);
    tma_prefetch_desc(&p.tm_sup);
    tma_prefetch_desc(&p.tm_down);
    tma_prefetch_desc(&p.tm_sdown);
    tma_prefetch_desc(&p.tm_up64);
    tma_prefetch_desc(&p.tm_x8);
    tma_prefetch_desc(&p.tm_sup64);
    tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  volatile int* abort = &sh.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // The up GEMM's token rows (this CTA's normed rows) are written by the
      // routing warps; until then those B loads wait in a queue (issue
      // order) while the weight loads go out.
      struct PendB {
        int stage, slot, x;
      };
      PendB pend[kStages * kKB] = {};
      int npend = 0;
      bool tok_ready = false;
      const int xrow = cta * kDecodeN;
      auto flush = [&](bool force) {
        if (!tok_ready && mbar_test_wait(&sh.tokens, 0)) {
          tok_ready = true;
          fence_proxy_async_global();
        }
        if (!tok_ready && !force) return;
        for (int j = 0; j < npend; ++j)
          tma_load_2d(tiles + pend[j].stage * kStageBytes + kKB * kABytes + pend[j].slot * kBBytes,
                      &p.tm_x, &sh.full[pend[j].stage], pend[j].x, xrow);
        npend = 0;
      };
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      // the weights are read once per launch: evict them first, keeping the
      // token rows, logits and the partial outputs in L2
      const uint64_t stream_policy = l2_policy_evict_first();
      // the routing warps' loads go out first (the routing decides when the
      // routed weights can stream)
      if (!mbar_wait(&sh.loads_out, 0, abort)) {
        record_timeout(p.status, abort);
        ok = false;
      }
      // nk <= kKB consecutive k-blocks into the next free stage: weight boxes
      // at x = ax, ax + 64, ... (and for up the token boxes at bx, bx + 64, ...)
      auto issue = [&](const CUtensorMap* map, int ax, int ay, int nk, bool up, int bx,
                       uint32_t abytes) -> bool {
        if (!mbar_test_wait(&sh.empty[stage], phase ^ 1u)) {
          const long long t0 = clock64();
          // try_wait suspends this thread (no issue slots taken from the
          // other warps) when no token load is pending; with pending loads
          // it polls the tokens barrier between short sleeps
          while (npend ? !mbar_test_wait(&sh.empty[stage], phase ^ 1u)
                       : !mbar_try_wait(&sh.empty[stage], phase ^ 1u)) {
            if (npend) {
              flush(false);
              __nanosleep(64);
            }
            if (*abort || clock64() - t0 > kWaitLimitCycles) {
              record_timeout(p.status, abort);
              return false;
            }
          }
        }
        uint8_t* sa = tiles + stage * kStageBytes;
        // (a token box holds MAXT rows: the MMA reads all 16 rows of the slot,
        // but rows past T only reach accumulator columns the epilogue drops)
        mbar_arrive_expect_tx(&sh.full[stage], uint32_t(nk * (up ? abytes + MAXT * 128 : abytes)));
        for (int i = 0; i < nk; ++i)
          tma_load_2d_hint(sa + i * kABytes, map, &sh.full[stage], ax + i * 64, ay, stream_policy);
        if (up) {
          if (npend) flush(false);
          for (int i = 0; i < nk; ++i) {
            if (tok_ready)
              tma_load_2d(sa + kKB * kABytes + i * kBBytes, &p.tm_x, &sh.full[stage], bx + i * 64,
                          xrow);
            else
              pend[npend++] = PendB{stage, i, bx + i * 64};
          }
        }
        ++issued;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      // FP8 units: one E4M3 weight box (two k-blocks; for up also the two
      // token boxes) into the next free staging slot, for the routing warps
      // to dequantise
      uint8_t* slots = tiles + kStagesF8 * kStageBytes;
      int fs = 0, issued8 = 0;
      uint32_t fph = 0;
      bool tok8 = false;
      auto issue8 = [&](const CUtensorMap* map, int ax, int ay, bool up, int bx) -> bool {
        if (!mbar_wait(&sh.f8empty[fs], fph ^ 1u, abort)) {
          record_timeout(p.status, abort);
          return false;
        }
        if (up && !tok8) {  // (complete since the routing; makes the rows visible to TMA)
          if (!mbar_wait(&sh.tokens, 0, abort)) {
            record_timeout(p.status, abort);
            return false;
          }
          fence_proxy_async_global();
          tok8 = true;
        }
        uint8_t* sl = slots + fs * kF8SlotBytes;
        // (the up's token rows: two f16 boxes for the dequantising path, one
        // E4M3 box of the same 128 elements under W8A8)
        mbar_arrive_expect_tx(&sh.f8full[fs],
                              uint32_t(kF8ABytes + (up ? (p.w8 ? 1 : kKB) * MAXT * 128 : 0)));
        tma_load_2d_hint(sl, map, &sh.f8full[fs], ax, ay, stream_policy);
        if (up && p.w8)
          tma_load_2d(sl + kF8ABytes, &p.tm_x8, &sh.f8full[fs], bx, xrow);
        else if (up)
          for (int i = 0; i < kKB; ++i)
            tma_load_2d(sl + kF8ABytes + i * kBBytes, &p.tm_x, &sh.f8full[fs], bx + i * 64, xrow);
        ++issued8;
        if (++fs == kF8Slots) {
          fs = 0;
          fph ^= 1u;
        }
        return true;
      };
      int m = 0;
      bool routed = false;
      for (int s = 0; ok; ++s) {
        int kind, n;
        if (!step_of(un, m, s, &kind, &n)) {
          if (routed) break;
          // the routed units: wait for this CTA's routing (test_wait: the
          // pending token loads are this thread's to issue)
          const long long t0 = clock64();
          while (npend ? !mbar_test_wait(&sh.routed, 0) : !mbar_try_wait(&sh.routed, 0)) {
            if (npend) {
              flush(false);
              __nanosleep(64);
            }
            if (*abort || clock64() - t0 > kWaitLimitCycles) {
              ok = false;
              break;
            }
          }
          if (!ok || *abort) {
            record_timeout(p.status, abort);
            ok = false;
            break;
          }
          routed = true;
          un.N = un.nS + sh.U * un.nI;
          m = un.count();
          if (!step_of(un, m, s, &kind, &n)) break;
        }
        const UnitInfo f = unit_info(p, sh, un, n);
        if (conv) {  // FP8 routed unit (E4M3 boxes of 128 elements = two k-blocks)
          if (kind == 0) {
            for (int kb = 0; ok && kb < kbH; kb += kKB)
              ok = issue8(&p.tm_up, kb * 64, f.expert * p.I + f.row0, true, kb * 64);
          } else {
            for (int r = 0; ok && r < nH; ++r)
              ok = issue8(&p.tm_down, f.row0, f.expert * p.H + r * kBM, false, 0);
          }
        } else if (kind == 0) {  // up: W_up[rows] x tokens, K = H
          // (a unit of 64 rows loads 64-row boxes: the stage's other 64
          // A rows keep stale data, whose accumulator rows are not used)
          const bool half = f.row_end - f.row0 <= 64;
          const CUtensorMap* map = f.shared ? (half ? &p.tm_sup64 : &p.tm_sup)
                                            : (half ? &p.tm_up64 : &p.tm_up);
          const int ay = f.shared ? f.row0 : f.expert * p.I + f.row0;
          const uint32_t ab = half ? uint32_t(kABytes / 2) : uint32_t(kABytes);
          for (int kb = 0; ok && kb < kbH; kb += kKB)
            ok = issue(map, kb * 64, ay, min(kKB, kbH - kb), true, kb * 64, ab);
        } else {  // down: W_down[:, rows] for every 128-row block of H
          const CUtensorMap* map = f.shared ? &p.tm_sdown : &p.tm_down;
          const int nkk = down_kk(f);
          for (int r = 0; ok && r < nH; ++r)
            ok = issue(map, f.row0, (f.shared ? 0 : f.expert * p.H) + r * kBM, nkk, false, 0,
                       uint32_t(kABytes));
        }
      }
      // the remaining token loads (also on an abort, so that every issued
      // stage completes and can be drained)
      if (ok && npend) {
        const long long t0 = clock64();
        while (npend) {
          flush(false);
          if (npend && (*abort || clock64() - t0 > kWaitLimitCycles)) {
            record_timeout(p.status, abort);
            ok = false;
            break;
          }
        }
      }
      if (!ok) {
        flush(true);
        int s = stage;
        uint32_t ph = phase;
        const int n = issued < kStages ? issued : kStages;
        for (int i = 0; i < n; ++i) {
          if (--s < 0) {
            s = kStages - 1;
            ph ^= 1u;
          }
          int zero = 0;
          mbar_wait(&sh.full[s], ph, &zero);
        }
        // and the FP8 boxes in flight
        s = fs;
        ph = fph;
        const int n8 = issued8 < kF8Slots ? issued8 : kF8Slots;
        for (int i = 0; i < n8; ++i) {
          if (--s < 0) {
            s = kF8Slots - 1;
            ph ^= 1u;
          }
          int zero = 0;
          mbar_wait(&sh.f8full[s], ph, &zero);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(kBM, kDecodeN, 1, 1);    // BF16 x BF16 -> F32
      const uint32_t idesc_h = make_idesc(kBM, kDecodeN, 0, 0);  // F16 x F16 -> F32 (FP8 units' up)
      const uint32_t idesc_8 = make_idesc(kBM, kDecodeN, 0, 0);  // E4M3 x E4M3 -> F32 (W8A8)
      const bool w8 = conv && p.w8;  // (W8A8: the MMA reads the FP8 slots themselves)
      const uint8_t* slots = tiles + kStagesF8 * kStageBytes;
      int fs = 0;
      uint32_t fph = 0;
      // the next FP8 slot, once its boxes have landed; false on timeout
      auto slot_wait = [&]() -> bool {
        if (!mbar_wait(&sh.f8full[fs], fph, abort)) {
          record_timeout(p.status, abort);
          return false;
        }
        tc_fence_after();
        return true;
      };
      auto slot_release = [&]() {
        umma_commit(&sh.f8empty[fs]);
        if (++fs == kF8Slots) {
          fs = 0;
          fph ^= 1u;
        }
      };
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int m = 0;
      bool routed = false, any = false;
      for (int s = 0; ok; ++s) {
        int kind, n;
        if (!step_of(un, m, s, &kind, &n)) {
          if (routed) break;
          if (!mbar_wait(&sh.routed, 0, abort) || *abort) {
            record_timeout(p.status, abort);
            ok = false;
            break;
          }
          routed = true;
          un.N = un.nS + sh.U * un.nI;
          m = un.count();
          if (!step_of(un, m, s, &kind, &n)) break;
        }
        const UnitInfo f = unit_info(p, sh, un, n);
        const int b = n & 1;
        const uint32_t par = (n >> 1) & 1;
        any = true;
        if (kind == 0) {
          // up into accumulator b (free once the epilogue has read unit n - 2)
          if (!mbar_wait(&sh.tempty[b], par ^ 1u, abort)) {
            record_timeout(p.status, abort);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + uint32_t(b * kDecodeN);
          if (w8) {  // one slot per two k-blocks: 128 E4M3 weights x 128 E4M3 token bytes
            for (int kb = 0; ok && kb < kbH; kb += kKB) {
              if (!slot_wait()) {
                ok = false;
                break;
              }
              const uint8_t* sl = slots + fs * kF8SlotBytes;
              const uint64_t ad = smem_desc_sw128(sl);
              const uint64_t bd = smem_desc_sw128(sl + kF8ABytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t koff = uint64_t((kk * 32) >> 4);
                umma_f8(d, ad + koff, bd + koff, idesc_8, (kb != 0 || kk != 0) ? 1u : 0u);
              }
              slot_release();
            }
            if (ok) umma_commit(&sh.tfull[b]);
            continue;
          }
          for (int kb = 0; kb < kbH; kb += kKB) {
            if (!mbar_wait(&sh.full[stage], phase, abort)) {
              record_timeout(p.status, abort);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint8_t* sa = tiles + stage * kStageBytes;
            const int nk = min(kKB, kbH - kb);
            for (int i = 0; i < nk; ++i) {
              const uint64_t ad = smem_desc_sw128(sa + i * kABytes);
              const uint64_t bd = smem_desc_sw128(sa + kKB * kABytes + i * kBBytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t koff = uint64_t((kk * 32) >> 4);
                umma_f16(d, ad + koff, bd + koff, conv ? idesc_h : idesc,
                         (kb + i != 0 || kk != 0) ? 1u : 0u);
              }
            }
            umma_commit(&sh.empty[stage]);
            if (++stage == nst) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) umma_commit(&sh.tfull[b]);
        } else {
          // down: the unit's relu^2 rows (buffer b) against W_down[:, rows],
          // added into the H x 16 accumulator
          if (!mbar_wait(&sh.ufull[b], par, abort)) {
            record_timeout(p.status, abort);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* ub = ubufs + b * kUBytes;
          if (w8) {  // the unit's 128 K columns of each 128-row block of H in one slot
            for (int r = 0; ok && r < nH; ++r) {
              const uint32_t d = tmem_base + uint32_t((2 + r) * kDecodeN);
              if (!slot_wait()) {
                ok = false;
                break;
              }
              const uint64_t ad = smem_desc_sw128(slots + fs * kF8SlotBytes);
              const uint64_t bd = smem_desc_sw128(ub);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t koff = uint64_t((kk * 32) >> 4);
                umma_f8(d, ad + koff, bd + koff, idesc_8, (n != 0 || kk != 0) ? 1u : 0u);
              }
              slot_release();
            }
            if (ok) umma_commit(&sh.ufree[b]);
            continue;
          }
          const int nkk = down_kk(f);
          for (int r = 0; ok && r < nH; ++r) {
            const uint32_t d = tmem_base + uint32_t((2 + r) * kDecodeN);
            if (!mbar_wait(&sh.full[stage], phase, abort)) {
              record_timeout(p.status, abort);
              ok = false;
              break;
            }
            tc_fence_after();
            for (int kc = 0; kc < nkk; ++kc) {
              const uint64_t ad = smem_desc_sw128(tiles + stage * kStageBytes + kc * kABytes);
              const uint64_t bd = smem_desc_sw128(ub + kc * kBBytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t koff = uint64_t((kk * 32) >> 4);
                umma_f16(d, ad + koff, bd + koff, idesc, (n != 0 || kc != 0 || kk != 0) ? 1u : 0u);
              }
            }
            umma_commit(&sh.empty[stage]);
            if (++stage == nst) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) umma_commit(&sh.ufree[b]);
        }
      }
      if (ok && any) umma_commit(&sh.down_done);
      umma_commit(&sh.drain);
      int zero = 0;
      mbar_wait(&sh.drain, 0, &zero);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int tid = threadIdx.x - 64;
    // the dry routing pass (see route_select), then the real one may start
    route_select(p, sh, tid, abort, kBarEpi, true);
    if (tid == 0) mbar_arrive(&sh.warm);
    // and the final reduction's (one source, one token, four rows)
    finish_slice(p, 1, 0, 4, tid, kEpiThreads, true);
    // the factors r_t of the token rows (published with the rows)
    if (lane == 0 && !mbar_wait(&sh.tokens, 0, abort)) record_timeout(p.status, abort);
    __syncwarp();
    float rsc[kDecodeN];
#pragma unroll
    for (int c = 0; c < kDecodeN; ++c) rsc[c] = c < MAXT && c < p.T ? sh.rs[c] : 0.f;
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int rloc = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (uint32_t(q * 32) << 16);
    bool ok = true, routed = false;
    int m = un.shared_first() ? 1 : 0;
    // the tokens this CTA's units reach: its partial output is exactly zero
    // in every other column (their relu^2 rows are zero), which it need not add
    uint32_t tmask = 0;
    const bool w8 = conv && p.w8;
    int e8 = 0;  // (W8A8: the expert of the CTA's one unit)
    for (int n = 0; ok; ++n) {
      if (n >= m) {
        if (routed) break;
        // the routed units (and their routing weights): wait for the routing
        if (lane == 0 && !mbar_wait(&sh.routed, 0, abort)) record_timeout(p.status, abort);
        __syncwarp();
        if (epi_stop(sh, tid)) {
          ok = false;
          break;
        }
        routed = true;
        un.N = un.nS + sh.U * un.nI;
        m = un.count();
        if (n >= m) break;
      }
      const UnitInfo f = unit_info(p, sh, un, n);
      const int b = n & 1;
      const uint32_t par = (n >> 1) & 1;
      e8 = f.expert;
#pragma unroll
      for (int c = 0; c < MAXT; ++c)
        if (c < p.T && (f.shared || sh.seg_w[f.slot][c] != 0.f)) tmask |= 1u << c;
      const bool valid = f.row0 + rloc < f.row_end;
      // an FP8 unit's up runs on the unscaled E4M3 values: its row's scale
      // (loaded while the up runs)
      const float srow = conv && !f.shared && valid
                             ? p.up_scale[size_t(f.expert) * p.I + f.row0 + rloc]
                             : 1.f;
      // the up accumulator of unit n
      if (lane == 0 && !mbar_wait(&sh.tfull[b], par, abort)) record_timeout(p.status, abort);
      __syncwarp();
      if (epi_stop(sh, tid)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[16];
      tmem_ld_32x32b_x16(lane_base + uint32_t(b * kDecodeN), r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tempty[b]);
      // relu^2 times the routing weight (1 for the shared expert); rows past
      // the matrix (an expert's last tile) and tokens past T are zero
      float v[kDecodeN];
      const float s8 = w8 ? sh.x8s : 1.f;  // (W8A8: the token row's E4M3 scale)
#pragma unroll
      for (int c = 0; c < kDecodeN; ++c) {
        const float w = f.shared ? (c < p.T ? 1.f : 0.f) : sh.seg_w[f.slot][c];
        const float a = __uint_as_float(r[c]) * rsc[c] * srow * s8;
        v[c] = valid && w != 0.f ? (a > 0.f ? a * a : 0.f) * w : 0.f;
      }
      // W8A8 (one token): the relu^2 rows as E4M3 with one scale, max |v| / 448
      float inv8 = 1.f;
      if (w8) {
        const float um = warp_max(fabsf(v[0]));
        if (lane == 0) sh.amax8[warp & 3] = um;
        named_barrier(kBarEpi, kEpiThreads);
        const float mx = fmaxf(fmaxf(sh.amax8[0], sh.amax8[1]), fmaxf(sh.amax8[2], sh.amax8[3]));
        const float su = mx > 0.f ? mx / 448.f : 1.f;
        inv8 = 1.f / su;
        if (tid == 0) sh.u8s = su;
      }
      // buffer b is free once unit n - 2's down MMAs have completed
      if (n >= 2) {
        if (lane == 0 && !mbar_wait(&sh.ufree[b], ((n - 2) >> 1) & 1, abort))
          record_timeout(p.status, abort);
        __syncwarp();
        if (epi_stop(sh, tid)) {
          ok = false;
          break;
        }
      }
      if (w8) {
        // K-major E4M3 token rows of 128 bytes (128-byte swizzle: 16-byte chunk
        // j of row c at j ^ (c % 8)); row 0 is the token, the others zero
        uint8_t* ub = ubufs + b * kUBytes;
        const __nv_fp8x2_storage_t q2 = __nv_cvt_float2_to_fp8x2(
            make_float2(v[0] * inv8, 0.f), __NV_SATFINITE, __NV_E4M3);
#pragma unroll
        for (int c = 0; c < kDecodeN; ++c)
          ub[c * 128 + ((((rloc >> 4) ^ (c & 7)) << 4) | (rloc & 15))] =
              c == 0 ? uint8_t(q2 & 0xffu) : uint8_t(0);
      } else {
        store_u_row(ubufs + b * kUBytes, rloc, v);
      }
      fence_proxy_async_shared();  // generic writes -> tensor core reads
      named_barrier(kBarEpi, kEpiThreads);
      if (tid == 0) mbar_arrive(&sh.ufull[b]);
    }
    // this CTA's partial output (the H x 16 down accumulator, columns < T)
    // into the launch's fixed-point sum.  From four tokens on, the partial
    // goes to shared memory, token-major [T, H] (the ring is idle once every
    // down MMA has completed), and all warps issue the T x H adds below (at
    // T = 8 this shortens the tail by about 1 us); below four, the epilogue
    // warps add it themselves (the extra barrier would cost more)
    if (ok && m > 0) {
      if (lane == 0 && !mbar_wait(&sh.down_done, 0, abort)) record_timeout(p.status, abort);
      __syncwarp();
      if (!epi_stop(sh, tid)) {
        tc_fence_after();
        float* stagef = reinterpret_cast<float*>(tiles);
        // (below four tokens, where the CTAs finish at about the same time,
        // each starts at its own row tile rather than all adding to the
        // same addresses together)
        // (the MAXT token columns of kTilesPerWait row tiles per TMEM wait:
        // below four tokens the adds follow at once, and eight tiles per wait
        // took 0.7 us off the last CTA's tail; the staged path, which only
        // writes shared memory here, was 0.7 us slower that way at T = 4)
        constexpr int kTilesPerWait = kStagePartial ? 1 : 8;
        for (int i0 = 0; i0 < nH; i0 += kTilesPerWait) {
          uint32_t r[kTilesPerWait][MAXT];
#pragma unroll
          for (int g = 0; g < kTilesPerWait; ++g) {
            const int i = i0 + g;
            const int rt = kStagePartial ? i : (i + cta) % nH;
            if (i < nH) tmem_ld_32x32b_n<MAXT>(lane_base + uint32_t((2 + rt) * kDecodeN), r[g]);
          }
          tmem_ld_wait_regs(r);
#pragma unroll
          for (int g = 0; g < kTilesPerWait; ++g) {
            const int i = i0 + g;
            const int rt = kStagePartial ? i : (i + cta) % nH;
            const int row = rt * kBM + rloc;
            if (i >= nH || row >= p.H) continue;
#pragma unroll
            for (int c = 0; c < MAXT; ++c) {
              if (!((tmask >> c) & 1u)) continue;
              // (W8A8: the down weight row's scale and the relu^2 rows' scale)
              const float sc8 =
                  w8 ? p.down_scale[size_t(e8) * p.H + row] * sh.u8s : 1.f;
              if constexpr (kStagePartial)
                stagef[c * p.H + row] = __uint_as_float(r[g][c]) * sc8;
              else
                add_partial(p.ws, size_t(c) * p.H + row, __uint_as_float(r[g][c]) * sc8);
            }
          }
        }
        tc_fence_before();
        named_barrier(kBarEpi, kEpiThreads);
        if (tid == 0) {
          if constexpr (kStagePartial) {
            sh.partial_tokens = tmask;
            sh.has_partial = 1;
          } else
            red_release_add(p.ws.sync + kPartialsDone, 1u);
        }
      }
    }
  } else {
    // ------------------------------------------------------------- routing
    const int rt = threadIdx.x - 192;
    route_logits<MAXT, F8>(p, sh, rt, rl, conv);
    const bool routed_ok = route_select(p, sh, rt, abort, kBarRoute, false);
    if (rt == 0) mbar_arrive(&sh.routed);  // (also on failure: the waiters then see abort)
    if (conv && !p.w8 && routed_ok && !*abort) {
      Units ur = un;
      ur.N = un.nS + sh.U * un.nI;
      dequant_stages(p, sh, ur, tiles, rt, abort);
    }
  }

  // ----------------------------------------------- reduction and wind down
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  // this CTA's partial output, staged by the epilogue warps, into the
  // launch's fixed-point sum: every warp issues the T x H atomic adds
  if (kStagePartial && sh.has_partial) {
    const float* stagef = reinterpret_cast<const float*>(tiles);
    const uint32_t tm = sh.partial_tokens;
    for (int c = 0; c < p.T; ++c) {
      if (!((tm >> c) & 1u)) continue;
      for (int i = threadIdx.x; i < p.H; i += kThreads)
        add_partial(p.ws, size_t(c) * p.H + i, stagef[c * p.H + i]);
    }
    __syncthreads();
    if (threadIdx.x == 0) red_release_add(p.ws.sync + kPartialsDone, 1u);
  }
  // Rows [r0, r0 + nr) of the output, once every CTA that had units has
  // added its partial and every CTA's logits are in (after that no CTA reads
  // hidden any more, so the rows can be overwritten).  (Thread 0 takes the
  // unit count from the slot table: only some roles have updated their own
  // copy of it.)
  const int n_units = un.nS + sh.U * un.nI;
  if (threadIdx.x == 0 && !*abort) {
    const unsigned active = unsigned(n_units < G ? n_units : G);
    if (!wait_counter(p.ws.sync + kPartialsDone, active, abort) ||
        !wait_counter(p.ws.sync + kRouteArrived, unsigned(G), abort))
      record_timeout(p.status, abort);
  }
  __syncthreads();
  if (!*abort) {
    const int R0 = reduce_rows(p.H, G);
    const int r0 = cta * R0;
    const int nr = min(p.H, r0 + R0) - r0;  // a multiple of 4: H is one of 64
    if (nr > 0) finish_slice(p, p.T, r0, nr, threadIdx.x, kThreads, false);
  }
  if (threadIdx.x == 0) {
    // the last CTA out resets the launch's synchronisation words: every
    // other CTA has passed its last wait on them
    __threadfence();
    sh.flag = atomicAdd(p.ws.sync + kExited, 1u) == unsigned(G - 1);
    if (sh.flag) {
      p.ws.sync[kRouteArrived] = 0u;
      p.ws.sync[kPartialsDone] = 0u;
      p.ws.sync[kExited] = 0u;
    }
  }
}

}  // namespace

bool fused_decode_supported(const moe_config& c, int grid) {
  // the routing warps hold a token row in kMaxChunks 8-element chunks each;
  // the H x 16 down accumulator fits next to the two up accumulators in TMEM;
  // FP8 routed experts (with row scales) need a BF16 shared expert, whose
  // units then take CTAs of their own: at most half of the grid
  const int nS = (c.shared_inter + kSharedUnit - 1) / kSharedUnit;
  const bool experts_ok = c.expert_wdtype == MOE_WEIGHTS_BF16 ||
                          (c.expert_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE && 2 * nS <= grid);
  return grid > 0 && c.latent_size == 0 && experts_ok && c.shared_wdtype == MOE_WEIGHTS_BF16 &&
         c.hidden_size <= kMaxChunks * kRouteThreads * 8 &&
         (c.hidden_size + kBM - 1) / kBM <= kMaxRowTiles;
}

namespace {

template <int MAXT, bool F8>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(decode_fused_kernel<MAXT, F8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kSmemOf(F8) + int(sizeof(Shared)));
}

template <bool F8>
cudaError_t launch_bucket(const cudaLaunchConfig_t& cfg, int T, const FusedParams& p) {
  if (T <= 1) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<1, F8>, p);
  if (T <= 2) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<2, F8>, p);
  if (T <= 4) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<4, F8>, p);
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel<8, F8>, p);
}

}  // namespace

cudaError_t prepare_fused_decode() {
  cudaError_t e;
  if ((e = set_smem<1, false>()) != cudaSuccess || (e = set_smem<2, false>()) != cudaSuccess ||
      (e = set_smem<4, false>()) != cudaSuccess || (e = set_smem<8, false>()) != cudaSuccess ||
      (e = set_smem<1, true>()) != cudaSuccess || (e = set_smem<2, true>()) != cudaSuccess ||
      (e = set_smem<4, true>()) != cudaSuccess || (e = set_smem<8, true>()) != cudaSuccess)
    return e;
  return cudaSuccess;
}

cudaError_t launch_fused_decode(const FusedDecodeArgs& a, cudaStream_t stream) {
  const moe_config& c = *a.cfg;
  if (!fused_decode_supported(c, a.grid) || a.T < 1 || a.T > kDecodeMaxT)
    return cudaErrorInvalidValue;
  const bool f8 = c.expert_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE;
  if (f8 && (!a.w->up_scale || !a.w->down_scale)) return cudaErrorInvalidValue;
  FusedParams p;
  p.tm_up = *a.tm_up;
  p.tm_sup = *a.tm_sup;
  p.tm_down = *a.tm_down;
  p.tm_sdown = *a.tm_sdown;
  p.tm_up64 = *a.tm_up64;
  p.tm_x8 = *a.tm_x8;
  p.tm_sup64 = *a.tm_sup64;
  const int bucket = a.T <= 1 ? 0 : a.T <= 2 ? 1 : a.T <= 4 ? 2 : 3;
  p.tm_x = *a.tm_x[bucket];
  p.hidden = a.hidden;
  p.residual = a.residual;
  p.out = a.out ? a.out : a.hidden;
  p.norm_w = static_cast<const bf16*>(a.w->norm_w);
  p.gate_w = static_cast<const bf16*>(a.w->gate_w);
  p.gate_bias = a.w->gate_bias;
  p.up_scale = f8 ? a.w->up_scale : nullptr;
  p.down_scale = f8 ? a.w->down_scale : nullptr;
  p.T = a.T;
  p.H = c.hidden_size;
  p.E = c.num_experts;
  p.k = c.top_k;
  p.I = c.moe_inter;
  p.S = c.shared_inter;
  p.eps = c.rms_eps;
  p.rsf = c.routed_scaling_factor;
  p.ws = *a.ws;
  p.status = a.status;
  // W8A8 (the note at kSharedUnit): one token chooses top_k distinct
  // experts; their routed units must fit on the CTAs beside the shared ones
  {
    const int nS = (c.shared_inter + kSharedUnit - 1) / kSharedUnit;
    const int nI = (c.moe_inter + kBM - 1) / kBM;
    p.w8 = f8 && a.T == 1 && c.top_k * nI <= a.grid - nS ? 1 : 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemOf(f8) + sizeof(Shared);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return f8 ? launch_bucket<true>(cfg, a.T, p) : launch_bucket<false>(cfg, a.T, p);
}

}  // namespace moe
