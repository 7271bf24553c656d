// C ABI of the MoE FFN layer (include/moe_b200.h): argument validation,
// workspace, TMA descriptors and the launch sequence of both paths.
//
// Prefill path (any T), after NemotronMoeLayer `prefill` and MoeLayer
// `forward_prefill`:
//   rmsnorm -> router GEMM with fused sigmoid top-k (+ LatentMoE fc1 in the
//   same launch) -> sort by expert -> gather -> grouped up GEMM + relu^2
//   (routed experts and shared expert in one launch) -> grouped down GEMM
//   (routed + shared) -> unpermute + weighted reduce + shared + residual
//   (direct) or latent reduce -> fc2 GEMM with shared + residual blend.
// Decode path (T <= 8): decode.cu.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>

#include "../../include/moe_b200.h"
#include "decode.h"
#include "moe_internal.h"

using moe::GemmParams;
using bf16 = __nv_bfloat16;

namespace {

constexpr uint32_t kMagic = 0x4D6F4542u;  // "MoEB"

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D K-major operand map: inner = K extent (elements), rows, row stride in
// bytes; box = 128 bytes of K x box_rows rows, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, bool byte_elems, uint64_t inner, uint64_t rows,
              uint64_t row_stride_bytes, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {byte_elems ? 128u : 64u, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, byte_elems ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The device address of page-locked host memory the device can address
// (16-byte aligned), or null.
void* mapped_device_pointer(const void* host) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || !a.devicePointer || !aligned16(a.devicePointer))
    return nullptr;
  return a.devicePointer;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

// Output columns per tile of the prefill up and down launches.  A CTA
// streams 16 KB of A and BN x 128 B of B per 128-byte k-block; BN = 256
// carries twice the tensor work of BN = 128 for 1.5x the bytes, which is
// what the launches' in-flight depth (4 stages, 192 KB) can sustain.  Narrow
// layers (N < 512 in a launch) keep BN = 128, which wastes fewer columns.
inline int prefill_bn(int n_routed, int n_shared) {
  return (n_routed >= 512 && n_shared >= 512) ? 256 : 128;
}

struct moe_handle {
  uint32_t magic;
  moe_config cfg;
  moe_weights w;
  int device;
  int num_sms;
  int D;           // routed-expert width
  bool fp8;         // routed experts E4M3
  bool shared_fp8;  // shared expert E4M3
  bool latent_fp8;  // fc1 / fc2 E4M3
  bool need_nq;     // some GEMM reads the E4M3 copy of the normed tokens
  int gate_bn;     // router GEMM tile width (>= E)
  int last_launches;
  void* const* stage_events;  // profiling: caller-owned cudaEvent_t array
  int n_stage_events;
  int last_tokens;    // num_tokens of the last forward
  bool last_decode;   // whether it took the decode path
  // workspace
  void* ws;
  size_t ws_bytes;
  bf16* gate_a;    // [Tm, 2H]: normed bf16 rows in the first H columns
  bf16* gate_w2;   // [E, 2H]: the gate with the norm weight folded in, BF16 hi | lo (set at create)
  float* rs;       // [Tm]: each token's RMSNorm factor rsqrt(mean x^2 + eps)
  int32_t* idx;    // [Tm*k]
  float* wts;      // [Tm*k]  (immediately after idx, as the pages' scratch layout)
  int32_t* off;    // [E+1]
  int2* tiles;     // [Rm/128 + E]
  float* topk_part;        // [sms * 128, E] router split-K partial logits
  int32_t* expert_hist;    // [ceil(Tm/128), E]
  int32_t* n_mtiles;
  int32_t* status;
  int32_t* sched;  // [4] dynamic tile schedule counters of the up and down launches
  int32_t* perm;   // [Rm]
  int32_t* inv;    // [Rm]
  bf16* z;         // [Tm, L]   latent fc1 output
  bf16* xs;        // [Rm, D]   sorted expert inputs
  bf16* u;         // [Rm, I]   relu^2(up)
  bf16* v;         // [Tm, S]   shared relu^2(up)
  bf16* y;         // [Rm, D]   routed expert outputs (sorted order)
  float* s;        // [Tm, H]   shared expert output
  bf16* m;         // [Tm, L]   latent weighted sum
  bf16* stage_h;   // [Tm, H]   host-path staging
  bf16* stage_r;   // [Tm, H]
  // FP8 experts: E4M3 activations with one float scale per row
  uint8_t* nq;       // [Tm, H]   normed tokens
  float* nq_scale;   // [Tm]
  float* xs_scale;   // [Rm]      scale of each sorted row (xs holds E4M3 bytes)
  unsigned* u_amax;  // [Rm]      running row max of relu^2(up) (float bits)
  uint8_t* uq;       // [Rm, I]   E4M3 relu^2(up)
  float* u_scale;    // [Rm]
  unsigned* v_amax;  // [Tm]      FP8 shared expert: running row max of relu^2(up)
  uint8_t* vq;       // [Tm, S]   E4M3 shared relu^2(up)
  float* v_scale;    // [Tm]
  uint8_t* mq;       // [Tm, L]   FP8 fc2: E4M3 latent weighted sum
  float* m_scale;    // [Tm]
  moe::FusedWorkspace dec;
  // tensor maps
  CUtensorMap tm_gate_b, tm_fc1_a, tm_fc1_b;
  CUtensorMap tm_up_a, tm_up_b, tm_sup_a, tm_sup_b;
  CUtensorMap tm_down_a, tm_down_b, tm_sdown_a, tm_sdown_b;
  // the same weights with up_bn / down_bn-row boxes (B operand of the
  // prefill launches; the decode launches read them as the 128-row A operand)
  CUtensorMap tm_up_w, tm_sup_w, tm_down_w, tm_sdown_w;
  // the up weights with 64-row boxes (the decode launch's units of 64 rows)
  CUtensorMap tm_up_b64, tm_sup_b64;
  int up_bn, down_bn;
  CUtensorMap tm_fc2_a, tm_fc2_b;
  CUtensorMap tm_dec_x[4];  // decode token rows, one 16-row block per CTA; boxes of 1, 2, 4, 8 rows
  CUtensorMap tm_dec_x8;    // the E4M3 token rows of the one-token FP8 launch, one-row boxes
};

namespace {

moe_status check_handle(const moe_handle* h) {
  return (h && h->magic == kMagic) ? MOE_OK : MOE_ERR_INVALID_HANDLE;
}

// A valid handle whose device is the current one: its workspace, weights
// and tensor maps live on that device, so a call made while another device
// is current is refused before anything is enqueued.
moe_status check_handle_device(const moe_handle* h) {
  moe_status st = check_handle(h);
  if (st != MOE_OK) return st;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) return MOE_ERR_DEVICE;
  return MOE_OK;
}

moe_status validate_config(const moe_config* c) {
  if (c->hidden_size <= 0 || c->num_experts <= 0 || c->moe_inter <= 0 || c->shared_inter <= 0 ||
      c->latent_size < 0 || c->max_tokens < 1)
    return MOE_ERR_INVALID_CONFIG;
  if (c->top_k < 1 || c->top_k > c->num_experts || c->top_k > MOE_MAX_TOP_K ||
      c->num_experts > MOE_MAX_EXPERTS)
    return MOE_ERR_INVALID_CONFIG;
  if (c->hidden_size % 64 || c->moe_inter % 64 || c->shared_inter % 64 || c->latent_size % 64)
    return MOE_ERR_INVALID_CONFIG;
  if (!(c->rms_eps >= 0.f) || !std::isfinite(c->rms_eps) ||
      !std::isfinite(c->routed_scaling_factor))
    return MOE_ERR_INVALID_CONFIG;
  for (int32_t dt : {c->expert_wdtype, c->shared_wdtype, c->latent_wdtype})
    if (dt != MOE_WEIGHTS_BF16 && dt != MOE_WEIGHTS_FP8_E4M3_ROWSCALE)
      return MOE_ERR_INVALID_CONFIG;
  // FP8 routed experts are wired for the direct layer (their input rows are
  // the E4M3 normed tokens)
  if (c->expert_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE && c->latent_size > 0)
    return MOE_ERR_INVALID_CONFIG;
  // row counts of the stacked expert maps and tile tables must fit in int32
  const long long D = c->latent_size ? c->latent_size : c->hidden_size;
  const long long R = 1ll * c->max_tokens * c->top_k;
  if (1ll * c->num_experts * c->moe_inter > (1ll << 31) - 1 ||
      1ll * c->num_experts * D > (1ll << 31) - 1 || R * (D > c->moe_inter ? D : c->moe_inter) >
                                                      (1ll << 40))
    return MOE_ERR_INVALID_CONFIG;
  return MOE_OK;
}

moe_status validate_weights(const moe_config* c, const moe_weights* w) {
  const bool fp8 = c->expert_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE;
  const void* req[] = {w->norm_w, w->gate_w, w->up_w, w->down_w, w->shared_up_w, w->shared_down_w};
  for (const void* p : req)
    if (!p) return MOE_ERR_NULL_POINTER;
  if (fp8 && (!w->up_scale || !w->down_scale)) return MOE_ERR_NULL_POINTER;
  if (c->shared_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE &&
      (!w->shared_up_scale || !w->shared_down_scale))
    return MOE_ERR_NULL_POINTER;
  if (c->latent_size > 0 && (!w->fc1_w || !w->fc2_w)) return MOE_ERR_NULL_POINTER;
  if (c->latent_size > 0 && c->latent_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE &&
      (!w->fc1_scale || !w->fc2_scale))
    return MOE_ERR_NULL_POINTER;
  const void* all[] = {w->norm_w, w->gate_w, w->gate_bias, w->up_w, w->down_w, w->up_scale,
                       w->down_scale, w->shared_up_w, w->shared_down_w, w->fc1_w, w->fc2_w,
                       w->shared_up_scale, w->shared_down_scale, w->fc1_scale, w->fc2_scale};
  for (const void* p : all)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

struct Carver {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off = round_up(off + count * sizeof(T), 256);
    return p;
  }
};

void carve(moe_handle* h, char* base) {
  const moe_config& c = h->cfg;
  const size_t Tm = c.max_tokens, k = c.top_k, E = c.num_experts, H = c.hidden_size;
  const size_t Rm = Tm * k, D = h->D, I = c.moe_inter, S = c.shared_inter, L = c.latent_size;
  Carver cv{base};
  h->gate_a = cv.take<bf16>(Tm * 2 * H);
  h->gate_w2 = cv.take<bf16>(size_t(E) * 2 * H);
  h->rs = cv.take<float>(Tm);
  h->idx = cv.take<int32_t>(Rm);
  h->wts = cv.take<float>(Rm);
  h->off = cv.take<int32_t>(E + 1);
  h->tiles = cv.take<int2>(Rm / moe::kBM + E + 1);
  h->topk_part = cv.take<float>(size_t(h->num_sms) * moe::kBM * E);
  h->expert_hist = cv.take<int32_t>((Tm + moe::kBM - 1) / moe::kBM * E);
  h->n_mtiles = cv.take<int32_t>(1);
  h->status = cv.take<int32_t>(1);
  h->sched = cv.take<int32_t>(4);
  h->perm = cv.take<int32_t>(Rm);
  h->inv = cv.take<int32_t>(Rm);
  h->z = L ? cv.take<bf16>(Tm * L) : nullptr;
  h->xs = cv.take<bf16>(Rm * D);
  h->u = cv.take<bf16>(Rm * I);
  h->v = cv.take<bf16>(Tm * S);
  h->y = cv.take<bf16>(Rm * D);
  h->s = cv.take<float>(Tm * H);
  h->m = L ? cv.take<bf16>(Tm * L) : nullptr;
  h->stage_h = cv.take<bf16>(Tm * H);
  h->stage_r = cv.take<bf16>(Tm * H);
  if (h->need_nq) {
    h->nq = cv.take<uint8_t>(Tm * H);
    h->nq_scale = cv.take<float>(Tm);
  }
  if (h->fp8) {
    h->xs_scale = cv.take<float>(Rm);
    h->u_amax = cv.take<unsigned>(Rm);
    h->uq = cv.take<uint8_t>(Rm * I);
    h->u_scale = cv.take<float>(Rm);
  }
  if (h->shared_fp8) {
    h->v_amax = cv.take<unsigned>(Tm);
    h->vq = cv.take<uint8_t>(Tm * S);
    h->v_scale = cv.take<float>(Tm);
  }
  if (L && h->latent_fp8) {
    h->mq = cv.take<uint8_t>(Tm * L);
    h->m_scale = cv.take<float>(Tm);
  }
  moe::carve_fused(&h->dec, c, h->num_sms, [&](size_t bytes) { return cv.take<char>(bytes); });
  h->ws_bytes = cv.off;
}

bool build_maps(moe_handle* h) {
  const moe_config& c = h->cfg;
  const uint64_t Tm = c.max_tokens, E = c.num_experts, H = c.hidden_size;
  const uint64_t Rm = Tm * c.top_k, D = h->D, I = c.moe_inter, S = c.shared_inter,
                 L = c.latent_size;
  const bool f8 = h->fp8, sf8 = h->shared_fp8, lf8 = h->latent_fp8;
  const uint64_t eb = f8 ? 1 : 2;   // bytes per routed-expert operand element
  const uint64_t sb = sf8 ? 1 : 2;  // shared expert
  const uint64_t lb = lf8 ? 1 : 2;  // fc1 / fc2
  bool ok = true;
  // router: A = [hi | lo] (K = 2H), B = gate [E, H] (k wraps at H)
  ok &= make_map(&h->tm_gate_b, h->gate_w2, false, 2 * H, E, 2 * H * 2, h->gate_bn);
  if (L) {  // FP8 fc1 / fc2 read the E4M3 normed tokens / latent sums
    if (lf8)
      ok &= make_map(&h->tm_fc1_a, h->nq, true, H, Tm, H, moe::kBM);
    else
      ok &= make_map(&h->tm_fc1_a, h->gate_a, false, H, Tm, 2 * H * 2, moe::kBM);
    ok &= make_map(&h->tm_fc1_b, h->w.fc1_w, lf8, H, L, H * lb, h->gate_bn);
    ok &= make_map(&h->tm_fc2_a, lf8 ? static_cast<const void*>(h->mq) : h->m, lf8, L, Tm,
                   L * lb, moe::kBM);
    ok &= make_map(&h->tm_fc2_b, h->w.fc2_w, lf8, L, H, L * lb, 128);
  }
  // grouped up: routed A = xs [Rm, D], B = up [E*I, D]; shared A = normed, B = [S, H]
  ok &= make_map(&h->tm_up_a, h->xs, f8, D, Rm, D * eb, moe::kBM);
  ok &= make_map(&h->tm_up_b, h->w.up_w, f8, D, E * I, D * eb, 128);
  if (sf8)
    ok &= make_map(&h->tm_sup_a, h->nq, true, H, Tm, H, moe::kBM);
  else
    ok &= make_map(&h->tm_sup_a, h->gate_a, false, H, Tm, 2 * H * 2, moe::kBM);
  ok &= make_map(&h->tm_sup_b, h->w.shared_up_w, sf8, H, S, H * sb, 128);
  ok &= make_map(&h->tm_up_b64, h->w.up_w, f8, D, E * I, D * eb, 64);
  ok &= make_map(&h->tm_sup_b64, h->w.shared_up_w, sf8, H, S, H * sb, 64);
  // grouped down: routed A = u [Rm, I], B = down [E*D, I]; shared A = v, B = [H, S]
  ok &= make_map(&h->tm_down_a, f8 ? static_cast<const void*>(h->uq) : h->u, f8, I, Rm, I * eb,
                 moe::kBM);
  ok &= make_map(&h->tm_down_b, h->w.down_w, f8, I, E * D, I * eb, 128);
  ok &= make_map(&h->tm_sdown_a, sf8 ? static_cast<const void*>(h->vq) : h->v, sf8, S, Tm,
                 S * sb, moe::kBM);
  ok &= make_map(&h->tm_sdown_b, h->w.shared_down_w, sf8, S, H, S * sb, 128);
  h->up_bn = prefill_bn(I, S);
  h->down_bn = prefill_bn(D, H);
  ok &= make_map(&h->tm_up_w, h->w.up_w, f8, D, E * I, D * eb, h->up_bn);
  ok &= make_map(&h->tm_sup_w, h->w.shared_up_w, sf8, H, S, H * sb, h->up_bn);
  ok &= make_map(&h->tm_down_w, h->w.down_w, f8, I, E * D, I * eb, h->down_bn);
  ok &= make_map(&h->tm_sdown_w, h->w.shared_down_w, sf8, S, H, S * sb, h->down_bn);
  if (moe::fused_decode_supported(c, h->num_sms)) {
    for (int b = 0; b < 4; ++b)
      ok &= make_map(&h->tm_dec_x[b], h->dec.x16, false, H, uint64_t(h->num_sms) * moe::kDecodeN,
                     H * 2, 1u << b);
    ok &= make_map(&h->tm_dec_x8, h->dec.x8, true, H, uint64_t(h->num_sms) * moe::kDecodeN, H, 1);
  }
  return ok;
}

moe::GemmClass dense_class(int K, int N, int rows, int epi, void* out, int ldo, int bn) {
  moe::GemmClass c{};
  c.K = K;
  c.N = N;
  c.ntiles = (N + bn - 1) / bn;
  c.rows = rows;
  c.mtiles = (rows + moe::kBM - 1) / moe::kBM;
  c.epi = epi;
  c.out = out;
  c.ldo = ldo;
  return c;
}

#define MOE_TRY(expr)                                  \
  do {                                                 \
    cudaError_t _e = (expr);                           \
    if (_e != cudaSuccess) return MOE_ERR_CUDA;        \
  } while (0)

// Norm + router GEMM with fused top-k (+ fc1 for LatentMoE).  When the
// token tiles alone would leave most SMs idle, the router's K (2H) is split
// so that tiles x splits fill the SMs left by the other class (or, when fc1
// fills them, into pieces shorter than fc1's tiles): every split stores
// fp32 partial logits and a second kernel sums them in split order and
// selects (one warp per token).
moe_status enqueue_route(moe_handle* h, const bf16* hidden, bf16* residual, int T,
                         bool with_fc1, cudaStream_t st, moe::LaunchLog* log) {
  const moe_config& c = h->cfg;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  // The router fused with the RMSNorm (NemotronMoeLayer `prefill`: the gate
  // runs on the normed rows): the raw rows x, read twice along K (the A
  // coordinate wraps at H), times [G'hi | G'lo] with G' = G * norm_w; each
  // token's logits are then r * (G' . x) = G . n, r applied in the epilogue.
  // Only the epilogue needs the RMSNorm launch (its factors r), so the
  // router's loads and MMAs start before that launch ends.
  if (!make_map(&p.tmA[0], hidden, false, c.hidden_size, T, c.hidden_size * 2, moe::kBM))
    return MOE_ERR_CUDA;
  p.tmB[0] = h->tm_gate_b;
  p.cls[0] = dense_class(2 * c.hidden_size, c.num_experts, T, moe::EPI_TOPK, nullptr, 0,
                         h->gate_bn);
  p.cls[0].ntiles = 1;
  p.cls[0].a_kwrap = c.hidden_size;
  p.topk_rs = h->rs;
  p.nclasses = 1;
  if (with_fc1 && c.latent_size > 0) {
    p.tmA[1] = h->tm_fc1_a;
    p.tmB[1] = h->tm_fc1_b;
    p.cls[1] = dense_class(c.hidden_size, c.latent_size, T, moe::EPI_BF16, h->z, c.latent_size,
                           h->gate_bn);
    if (h->latent_fp8) {  // W8A8: acc * token scale * weight-row scale
      p.cls[1].fp8 = 1;
      p.cls[1].row_scale = h->nq_scale;
      p.cls[1].col_scale = h->w.fc1_scale;
    }
    p.nclasses = 2;
  }
  const int mt = p.cls[0].mtiles;
  int ks = 1;
  if (c.num_experts <= 256) {
    const int nk = (2 * c.hidden_size + 63) / 64;
    const int other = p.nclasses > 1 ? p.cls[1].mtiles * p.cls[1].ntiles : 0;
    ks = h->num_sms > other ? (h->num_sms - other) / mt : 1;
    if (other > 0) {
      // With LatentMoE fc1 in the launch, cut the router tiles (K = 2H) into
      // pieces of at most half fc1's K, so that no router tile is the
      // launch's long pole (more pieces when idle SMs allow).
      const int nko = (p.cls[1].K + (p.cls[1].fp8 ? 127 : 63)) / (p.cls[1].fp8 ? 128 : 64);
      const int cut = 2 * ((nk + nko - 1) / nko);
      if (ks < cut) ks = cut;
    }
    if (ks > h->num_sms / mt) ks = h->num_sms / mt;  // capacity of the partial logits
    ks = ks < 1 ? 1 : (ks > moe::kRouterMaxSplit ? moe::kRouterMaxSplit : ks);
    ks = ks > nk ? nk : ks;
    const int per = (nk + ks - 1) / ks;
    ks = (nk + per - 1) / per;  // every split non-empty
  }
  p.cls[0].ksplit = ks;
  // (fc1's operand is the normed rows: with it in the launch every warp waits)
  p.epi_wait = p.nclasses == 1;
  MOE_TRY(moe::launch_rmsnorm(hidden, static_cast<const bf16*>(h->w.norm_w), residual, h->gate_a,
                              h->rs, h->need_nq && with_fc1 ? h->nq : nullptr, h->nq_scale, T,
                              c.hidden_size, c.rms_eps, ks > 1 ? h->expert_hist : nullptr,
                              mt * c.num_experts, st));
  log->done(st);
  p.topk_part = h->topk_part;
  p.topk_rows_cap = mt * moe::kBM;
  p.expert_hist = h->expert_hist;
  p.gate_bias = h->w.gate_bias;
  p.top_k = c.top_k;
  p.num_experts = c.num_experts;
  p.rsf = c.routed_scaling_factor;
  p.topk_idx = h->idx;
  p.topk_w = h->wts;
  p.status = h->status;
  int W = mt * ks + (p.nclasses > 1 ? p.cls[1].mtiles * p.cls[1].ntiles : 0);
  const int grid = W < h->num_sms ? W : h->num_sms;
  MOE_TRY(moe::launch_grouped_gemm(p, h->gate_bn, grid, st, /*pdl=*/true));
  log->done(st);
  if (ks > 1) {
    MOE_TRY(moe::launch_router_reduce(h->topk_part, ks, mt * moe::kBM, T, c.num_experts,
                                      h->w.gate_bias, c.top_k, c.routed_scaling_factor, h->rs,
                                      h->idx, h->wts, h->expert_hist, st));
    log->done(st);
  }
  return MOE_OK;
}

moe_status enqueue_prefill(moe_handle* h, bf16* hidden, bf16* residual, int T, cudaStream_t st,
                           moe::LaunchLog* log) {
  const moe_config& c = h->cfg;
  const int H = c.hidden_size, k = c.top_k, E = c.num_experts, I = c.moe_inter,
            S = c.shared_inter, L = c.latent_size, D = h->D, R = T * k;
  moe_status rs = enqueue_route(h, hidden, residual, T, true, st, log);
  if (rs != MOE_OK) return rs;
  MOE_TRY(moe::launch_sort(h->idx, h->expert_hist, T, k, E, h->perm, h->inv, h->off, h->tiles,
                           h->n_mtiles, h->status, st));
  log->done(st);
  if (L)
    MOE_TRY(moe::launch_gather(h->z, size_t(L) * 2, h->perm, k, R, D * 2, h->xs, nullptr,
                               nullptr, st));
  else if (h->fp8)
    MOE_TRY(moe::launch_gather(h->nq, size_t(H), h->perm, k, R, D, h->xs, h->nq_scale,
                               h->xs_scale, st));
  else
    MOE_TRY(moe::launch_gather(h->gate_a, size_t(2 * H) * 2, h->perm, k, R, D * 2, h->xs,
                               nullptr, nullptr, st));
  log->done(st);

  // grouped up (+ relu^2): routed class 0 via the tile table, shared class 1
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.tmA[0] = h->tm_up_a;
  p.tmB[0] = h->tm_up_w;
  p.cls[0] = dense_class(D, I, 0, moe::EPI_RELU2_BF16, h->u, I, h->up_bn);
  if (h->fp8) {  // W8A8: acc * token scale * weight-row scale, row max for requantisation
    p.cls[0].fp8 = 1;
    p.cls[0].row_scale = h->xs_scale;
    p.cls[0].col_scale = h->w.up_scale;
    p.cls[0].row_amax = h->u_amax;
  }
  p.tmA[1] = h->tm_sup_a;
  p.tmB[1] = h->tm_sup_w;
  p.cls[1] = dense_class(H, S, T, moe::EPI_RELU2_BF16, h->v, S, h->up_bn);
  if (h->shared_fp8) {  // W8A8, row max of relu^2 for requantisation
    p.cls[1].fp8 = 1;
    p.cls[1].row_scale = h->nq_scale;
    p.cls[1].col_scale = h->w.shared_up_scale;
    p.cls[1].row_amax = h->v_amax;
  }
  p.nclasses = 2;
  p.tile_table = h->tiles;
  p.n_mtiles = h->n_mtiles;
  p.group_off = h->off;
  p.status = h->status;
  p.sched = h->sched;
  MOE_TRY(moe::launch_grouped_gemm(p, h->up_bn, h->num_sms, st));
  log->done(st);

  if (h->fp8 || h->shared_fp8) {  // E4M3 rows of relu^2(up), one scale per row
    MOE_TRY(moe::launch_quantize_rows(h->fp8 ? h->u : nullptr, h->u_amax, h->uq, h->u_scale,
                                      h->fp8 ? R : 0, I, h->shared_fp8 ? h->v : nullptr,
                                      h->v_amax, h->vq, h->v_scale, h->shared_fp8 ? T : 0, S,
                                      st));
    log->done(st);
  }

  // grouped down: routed -> y (bf16, sorted rows), shared -> s (f32)
  p.tmA[0] = h->tm_down_a;
  p.tmB[0] = h->tm_down_w;
  p.cls[0] = dense_class(I, D, 0, moe::EPI_BF16, h->y, D, h->down_bn);
  if (h->fp8) {
    p.cls[0].fp8 = 1;
    p.cls[0].row_scale = h->u_scale;
    p.cls[0].col_scale = h->w.down_scale;
  }
  p.tmA[1] = h->tm_sdown_a;
  p.tmB[1] = h->tm_sdown_w;
  p.cls[1] = dense_class(S, H, T, moe::EPI_F32, h->s, H, h->down_bn);
  if (h->shared_fp8) {
    p.cls[1].fp8 = 1;
    p.cls[1].row_scale = h->v_scale;
    p.cls[1].col_scale = h->w.shared_down_scale;
    p.cls[1].row_amax = nullptr;
  }
  p.sched = h->sched + 2;
  MOE_TRY(moe::launch_grouped_gemm(p, h->down_bn, h->num_sms, st));
  log->done(st);

  if (!L) {
    MOE_TRY(moe::launch_combine(h->y, h->inv, h->wts, h->s, residual, hidden, T, k, H, st));
    log->done(st);
    return MOE_OK;
  }
  MOE_TRY(moe::launch_latent_reduce(h->y, h->inv, h->wts, h->m, h->latent_fp8 ? h->mq : nullptr,
                                    h->m_scale, T, k, L, st));
  log->done(st);
  GemmParams q;
  std::memset(&q, 0, sizeof(q));
  q.tmA[0] = h->tm_fc2_a;
  q.tmB[0] = h->tm_fc2_b;
  q.cls[0] = dense_class(L, H, T, moe::EPI_BLEND, hidden, H, 128);
  if (h->latent_fp8) {
    q.cls[0].fp8 = 1;
    q.cls[0].row_scale = h->m_scale;
    q.cls[0].col_scale = h->w.fc2_scale;
  }
  q.nclasses = 1;
  q.blend_s = h->s;
  q.blend_res = residual;
  q.status = h->status;
  const int W = q.cls[0].mtiles * q.cls[0].ntiles;
  MOE_TRY(moe::launch_grouped_gemm(q, 128, W < h->num_sms ? W : h->num_sms, st));
  log->done(st);
  return MOE_OK;
}

// Decode path (T <= 8): one cooperative launch (decode_fused.cu) with the
// weights as the 128-row operand and the tokens as N = 16.
// Whether MOE_PATH_AUTO takes the decode launch.  With FP8 routed experts
// only one token does: there every routed unit has a CTA to itself, and the
// launch runs W8A8 on the E4M3 weights (47 us on B200 for the skewed FP8
// workload's layer, against 98 us on the prefill path).  From two tokens
// on it dequantises the weights in shared memory, which no longer pays
// (118 against 104 us at T = 2).
bool decode_preferred(const moe_handle* h, int T) {
  return T <= MOE_DECODE_MAX_TOKENS && moe::fused_decode_supported(h->cfg, h->num_sms) &&
         (h->cfg.expert_wdtype == MOE_WEIGHTS_BF16 || T == 1);
}

// out: where the output rows go (null: hidden, in place).
moe_status enqueue_decode(moe_handle* h, bf16* hidden, bf16* residual, int T, cudaStream_t st,
                          moe::LaunchLog* log, bf16* out = nullptr) {
  const moe_config& c = h->cfg;
  if (!moe::fused_decode_supported(c, h->num_sms) || T < 1 || T > MOE_DECODE_MAX_TOKENS)
    return MOE_ERR_INVALID_CONFIG;
  moe::FusedDecodeArgs a;
  a.cfg = &c;
  a.w = &h->w;
  a.ws = &h->dec;
  a.tm_up = &h->tm_up_b;      // routed up weights [E*I, H], 128-row boxes
  a.tm_sup = &h->tm_sup_b;    // shared up weights [S, H]
  a.tm_down = &h->tm_down_b;  // routed down weights [E*H, I]
  a.tm_sdown = &h->tm_sdown_b;
  a.tm_up64 = &h->tm_up_b64;  // the same up weights, 64-row boxes
  a.tm_sup64 = &h->tm_sup_b64;
  for (int b = 0; b < 4; ++b) a.tm_x[b] = &h->tm_dec_x[b];
  a.tm_x8 = &h->tm_dec_x8;
  a.hidden = hidden;
  a.residual = residual;
  a.out = out;
  a.T = T;
  a.grid = h->num_sms;
  a.status = h->status;
  MOE_TRY(moe::launch_fused_decode(a, st));
  log->done(st);
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_CONFIG: return "invalid configuration";
    case MOE_ERR_NULL_POINTER: return "required pointer is NULL";
    case MOE_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case MOE_ERR_TOKENS_OUT_OF_RANGE: return "num_tokens outside [1, max_tokens]";
    case MOE_ERR_OUT_OF_MEMORY: return "workspace allocation failed";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "no sm_100 device is current";
    case MOE_ERR_INVALID_HANDLE: return "invalid handle";
  }
  return "unknown status";
}

moe_status moe_create(const moe_config* config, const moe_weights* weights, moe_handle** out) {
  if (!out) return MOE_ERR_NULL_POINTER;
  *out = nullptr;
  if (!config || !weights) return MOE_ERR_NULL_POINTER;
  moe_status st = validate_config(config);
  if (st != MOE_OK) return st;
  st = validate_weights(config, weights);
  if (st != MOE_OK) return st;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_DEVICE;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_DEVICE;
  if (prop.major != 10) return MOE_ERR_DEVICE;

  moe_handle* h = new (std::nothrow) moe_handle();
  if (!h) return MOE_ERR_OUT_OF_MEMORY;
  h->magic = kMagic;
  h->cfg = *config;
  h->w = *weights;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->D = config->latent_size ? config->latent_size : config->hidden_size;
  h->fp8 = config->expert_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE;
  h->shared_fp8 = config->shared_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE;
  h->latent_fp8 = config->latent_size > 0 && config->latent_wdtype == MOE_WEIGHTS_FP8_E4M3_ROWSCALE;
  h->need_nq = (h->fp8 && config->latent_size == 0) || h->shared_fp8 || h->latent_fp8;
  h->gate_bn = config->num_experts <= 128 ? 128 : 256;

  carve(h, nullptr);
  void* ws = nullptr;
  if (cudaMalloc(&ws, h->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MOE_ERR_OUT_OF_MEMORY;
  }
  h->ws = ws;
  carve(h, static_cast<char*>(ws));
  if (cudaMemset(ws, 0, h->ws_bytes) != cudaSuccess || !build_maps(h) ||
      moe::prepare_grouped_gemm() != cudaSuccess || moe::prepare_fused_decode() != cudaSuccess ||
      moe::launch_prep_gate(static_cast<const bf16*>(h->w.gate_w),
                            static_cast<const bf16*>(h->w.norm_w), config->num_experts,
                            config->hidden_size, h->gate_w2, 0) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(ws);
    h->magic = 0;
    delete h;
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

moe_status moe_destroy(moe_handle* h) {
  moe_status st = check_handle(h);
  if (st != MOE_OK) return st;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != h->device) cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  cudaFree(h->ws);
  if (cur != h->device) cudaSetDevice(cur);
  h->magic = 0;
  delete h;
  return MOE_OK;
}

moe_status moe_forward_path(moe_handle* h, void* hidden, void* residual, int32_t num_tokens,
                            int32_t path, void* stream) {
  moe_status st = check_handle_device(h);
  if (st != MOE_OK) return st;
  if (!hidden || !residual) return MOE_ERR_NULL_POINTER;
  if (!aligned16(hidden) || !aligned16(residual)) return MOE_ERR_MISALIGNED;
  if (num_tokens < 1 || num_tokens > h->cfg.max_tokens) return MOE_ERR_TOKENS_OUT_OF_RANGE;
  if (path != MOE_PATH_AUTO && path != MOE_PATH_DECODE && path != MOE_PATH_PREFILL)
    return MOE_ERR_INVALID_CONFIG;
  if (path == MOE_PATH_DECODE && num_tokens > MOE_DECODE_MAX_TOKENS)
    return MOE_ERR_TOKENS_OUT_OF_RANGE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe::LaunchLog log;
  log.events = h->stage_events;
  log.nevents = h->n_stage_events;
  log.begin(s);
  const bool decode = path == MOE_PATH_DECODE ||
                      (path == MOE_PATH_AUTO && decode_preferred(h, num_tokens));
  if (decode) {
    st = enqueue_decode(h, static_cast<bf16*>(hidden), static_cast<bf16*>(residual), num_tokens,
                        s, &log);
  } else {
    st = enqueue_prefill(h, static_cast<bf16*>(hidden), static_cast<bf16*>(residual), num_tokens,
                         s, &log);
  }
  h->last_launches = log.count;
  h->last_tokens = num_tokens;
  h->last_decode = decode;
  return st;
}

moe_status moe_forward(moe_handle* h, void* hidden, void* residual, int32_t num_tokens,
                       void* stream) {
  return moe_forward_path(h, hidden, residual, num_tokens, MOE_PATH_AUTO, stream);
}

moe_status moe_forward_host(moe_handle* h, void* hidden_host, void* residual_host,
                            int32_t num_tokens, void* stream) {
  moe_status st = check_handle_device(h);
  if (st != MOE_OK) return st;
  if (!hidden_host) return MOE_ERR_NULL_POINTER;
  if (num_tokens < 1 || num_tokens > h->cfg.max_tokens) return MOE_ERR_TOKENS_OUT_OF_RANGE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = size_t(num_tokens) * h->cfg.hidden_size * sizeof(bf16);
  MOE_TRY(cudaMemcpyAsync(h->stage_h, hidden_host, bytes, cudaMemcpyHostToDevice, s));
  // Decode sizes with page-locked buffers the device can address: the
  // kernel writes the output rows (and the residual) into them itself, so
  // no copy back and no launch of one follow the forward.
  if (decode_preferred(h, num_tokens)) {
    void* out_dev = mapped_device_pointer(hidden_host);
    void* res_dev = out_dev && residual_host ? mapped_device_pointer(residual_host) : nullptr;
    if (out_dev && (!residual_host || res_dev)) {
      moe::LaunchLog log;
      log.events = h->stage_events;
      log.nevents = h->n_stage_events;
      log.begin(s);
      st = enqueue_decode(h, h->stage_h, res_dev ? static_cast<bf16*>(res_dev) : h->stage_r,
                          num_tokens, s, &log, static_cast<bf16*>(out_dev));
      h->last_launches = log.count;
      h->last_tokens = num_tokens;
      h->last_decode = true;
      return st;
    }
  }
  st = moe_forward(h, h->stage_h, h->stage_r, num_tokens, stream);
  if (st != MOE_OK) return st;
  MOE_TRY(cudaMemcpyAsync(hidden_host, h->stage_h, bytes, cudaMemcpyDeviceToHost, s));
  if (residual_host)
    MOE_TRY(cudaMemcpyAsync(residual_host, h->stage_r, bytes, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

moe_status moe_route(moe_handle* h, const void* hidden, int32_t num_tokens, int32_t* idx,
                     float* w, void* stream) {
  moe_status st = check_handle_device(h);
  if (st != MOE_OK) return st;
  if (!hidden || !idx || !w) return MOE_ERR_NULL_POINTER;
  if (!aligned16(hidden)) return MOE_ERR_MISALIGNED;
  if (num_tokens < 1 || num_tokens > h->cfg.max_tokens) return MOE_ERR_TOKENS_OUT_OF_RANGE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe::LaunchLog log;
  st = enqueue_route(h, static_cast<const bf16*>(hidden), h->stage_r, num_tokens, false, s,
                     &log);
  if (st != MOE_OK) return st;
  const size_t n = size_t(num_tokens) * h->cfg.top_k;
  MOE_TRY(cudaMemcpyAsync(idx, h->idx, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  MOE_TRY(cudaMemcpyAsync(w, h->wts, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
  h->last_launches = log.count;
  return MOE_OK;
}

moe_status moe_sort(moe_handle* h, const int32_t* idx, int32_t num_tokens, int32_t* perm,
                    int32_t* inv, int32_t* off, void* stream) {
  moe_status st = check_handle_device(h);
  if (st != MOE_OK) return st;
  if (!idx || !perm || !inv || !off) return MOE_ERR_NULL_POINTER;
  if (num_tokens < 1 || num_tokens > h->cfg.max_tokens) return MOE_ERR_TOKENS_OUT_OF_RANGE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(moe::launch_tile_hist(idx, num_tokens, h->cfg.top_k, h->cfg.num_experts,
                                h->expert_hist, h->status, s));
  MOE_TRY(moe::launch_sort(idx, h->expert_hist, num_tokens, h->cfg.top_k, h->cfg.num_experts,
                           perm, inv, off, h->tiles, h->n_mtiles, h->status, s));
  h->last_launches = 2;
  return MOE_OK;
}

moe_status moe_copy_routing(moe_handle* h, int32_t* idx, float* w, int32_t num_tokens,
                            void* stream) {
  moe_status st = check_handle_device(h);
  if (st != MOE_OK) return st;
  if (!idx || !w) return MOE_ERR_NULL_POINTER;
  if (num_tokens < 1 || num_tokens != h->last_tokens) return MOE_ERR_TOKENS_OUT_OF_RANGE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t n = size_t(num_tokens) * h->cfg.top_k;
  const int32_t* si = h->last_decode ? h->dec.idx : h->idx;  // written by decode_route
  const float* sw = h->last_decode ? h->dec.w : h->wts;
  MOE_TRY(cudaMemcpyAsync(idx, si, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  MOE_TRY(cudaMemcpyAsync(w, sw, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
  return MOE_OK;
}

moe_status moe_copy_sort(moe_handle* h, int32_t* perm, int32_t* inv, int32_t* off,
                         int32_t num_tokens, void* stream) {
  moe_status st = check_handle_device(h);
  if (st != MOE_OK) return st;
  if (!perm || !inv || !off) return MOE_ERR_NULL_POINTER;
  if (num_tokens < 1 || num_tokens != h->last_tokens) return MOE_ERR_TOKENS_OUT_OF_RANGE;
  if (h->last_decode) return MOE_ERR_INVALID_CONFIG;  // the decode path does not sort
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t R = size_t(num_tokens) * h->cfg.top_k;
  MOE_TRY(cudaMemcpyAsync(perm, h->perm, R * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  MOE_TRY(cudaMemcpyAsync(inv, h->inv, R * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  MOE_TRY(cudaMemcpyAsync(off, h->off, (h->cfg.num_experts + 1) * sizeof(int32_t),
                          cudaMemcpyDeviceToDevice, s));
  return MOE_OK;
}

moe_status moe_get_device_status(moe_handle* h, int32_t* status, void* stream) {
  moe_status st = check_handle_device(h);
  if (st != MOE_OK) return st;
  if (!status) return MOE_ERR_NULL_POINTER;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_TRY(cudaMemcpyAsync(status, h->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  MOE_TRY(cudaMemsetAsync(h->status, 0, sizeof(int32_t), s));
  MOE_TRY(cudaStreamSynchronize(s));
  if (*status != 0) {
    // A pass that gave up on a wait may have left its tile and schedule
    // counters mid-count, and partial sums in the decode accumulator: start
    // the next one from zero.
    MOE_TRY(cudaMemsetAsync(h->dec.sync, 0, 4 * sizeof(unsigned), s));
    MOE_TRY(cudaMemsetAsync(h->dec.acc, 0,
                            size_t(moe::kDecodeMaxT) * h->cfg.hidden_size * sizeof(long long), s));
    MOE_TRY(cudaMemsetAsync(h->dec.bad, 0, size_t(moe::kDecodeMaxT) * h->cfg.hidden_size, s));
    MOE_TRY(cudaMemsetAsync(h->sched, 0, 4 * sizeof(int32_t), s));
    MOE_TRY(cudaStreamSynchronize(s));
  }
  return MOE_OK;
}

moe_status moe_set_stage_events(moe_handle* h, void* const* events, int32_t count) {
  moe_status st = check_handle(h);
  if (st != MOE_OK) return st;
  if (count < 0 || (count > 0 && !events)) return MOE_ERR_NULL_POINTER;
  h->stage_events = count > 0 ? events : nullptr;
  h->n_stage_events = count;
  return MOE_OK;
}

int32_t moe_last_launch_count(const moe_handle* h) {
  return check_handle(h) == MOE_OK ? h->last_launches : -1;
}

int32_t moe_last_path(const moe_handle* h) {
  if (check_handle(h) != MOE_OK || h->last_tokens < 1) return -1;
  return h->last_decode ? MOE_PATH_DECODE : MOE_PATH_PREFILL;
}

}  // extern "C"
