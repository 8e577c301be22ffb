// libuno: host runtime and C ABI of the Psi-Spec decode iteration.
//
// One iteration per request (blog page "不砸掉重来，给自回归 LLM 装一对“扩散翅膀”：
// Uno 的无损加速之路", sections 一句话直觉 and Ψ-Spec 采样器：起草、验证、两种模式):
//   draft pass   rows [pending, MASK x B] at positions c..c+B, LoRA gated on
//                for the MASK rows -> logits (AR p_1 on row 0, q_i on row i)
//   draft_sample x_1 ~ p_1 (AR only), x_i ~ q_i for i = 2..B
//   verify pass  rows x_1..x_B at c+1..c+B, LoRA off -> p_2..p_{B+1}
//   spec_verify  accept prefix, residual redraw or bonus, commit
// Draft and verify share the paged KV cache: the draft pass writes the
// pending token's keys/values at position c (final) and scratch keys for the
// MASK rows at c+1..c+B, which the verify pass then overwrites.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/uno.h"
#include "attn_simt.cuh"
#include "common.cuh"
#include "gemm_simt.cuh"
#include "layers.cuh"
#include "sampling.cuh"

using namespace uno;

struct uno_ctx {
  uno_shape s{};
  int r = 0, B = 0, max_batch = 0, max_ctx = 0;
  float alpha = 0.f, lscale = 0.f;
  uint64_t seed = 0;
  cudaStream_t stream = nullptr;
  size_t esz = 4;  // element size of the model dtype

  // weights (borrowed)
  const void *embed = nullptr, *lm_head = nullptr, *final_norm = nullptr;
  std::vector<const void*> attn_norm, ffn_norm;
  std::vector<const void*> w[UNO_N_PROJ], lA[UNO_N_PROJ], lB[UNO_N_PROJ];

  // KV pool and request slots
  KvLayout kv{};
  void* kv_pool = nullptr;
  int32_t* d_page_table = nullptr;
  int32_t *d_cached = nullptr, *d_pending = nullptr;
  uint32_t* d_stream = nullptr;
  std::vector<int> free_pages;
  std::vector<int> slot_used;
  std::vector<int32_t> h_page_table;

  // activations (sized for M_max rows)
  int M_max = 0;
  float* x = nullptr;          // [M, d] fp32 residual
  void* xn = nullptr;          // [M, max(d, F)]
  void* qkv = nullptr;         // [M, (H + 2 Hkv) hd]
  void* attn = nullptr;        // [M, H hd]
  void* gu = nullptr;          // [M, 2F]
  void* U = nullptr;           // [M, 3r] LoRA intermediate
  int32_t *row_pos = nullptr, *row_slot = nullptr;
  float* row_gate = nullptr;
  float *cos_t = nullptr, *sin_t = nullptr;
  int max_pos = 0;

  // logits and sampler state
  float *logits_d = nullptr, *logits_v = nullptr;   // [max_batch, B+1, V], [max_batch, B, V]
  int32_t* drafts = nullptr;                        // [max_batch, B]
  float* lse_q = nullptr;                           // [max_batch, B]
  int nch = 1, ch = 1;
  float2* partial = nullptr;                        // [max_batch * 2B, nch]
  float* lse_ws = nullptr;                          // [max_batch * 2B]
  unsigned* row_counter = nullptr;                  // [max_batch * 2B]
  unsigned* req_counter = nullptr;                  // [max_batch]

  // attention split workspace
  float* att_ws = nullptr;
  size_t att_ws_floats = 0;
  unsigned* att_counters = nullptr;
  int att_groups_max = 0;

  int32_t* d_status = nullptr;
  int last_n_req = 0;
  std::string err;

  // profiling tap
  unsigned prof_mask = 0;
  int64_t prof_launches[UNO_K_N] = {};
  double prof_bytes[UNO_K_N] = {};
  struct ProfRec { int cls; cudaEvent_t a, b; };
  std::vector<ProfRec> prof_recs;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_next = 0;
};

namespace {
cudaEvent_t next_event(uno_ctx* c) {
  if (c->ev_next == c->ev_pool.size()) {
    cudaEvent_t e;
    cudaEventCreate(&e);
    c->ev_pool.push_back(e);
  }
  return c->ev_pool[c->ev_next++];
}

// Counts a launch of class `cls` and, when that class is profiled, brackets it
// with an event pair on the context stream.
struct Prof {
  uno_ctx* c;
  int cls;
  cudaEvent_t a = nullptr, b = nullptr;
  Prof(uno_ctx* c_, int cls_, double bytes) : c(c_), cls(cls_) {
    c->prof_launches[cls]++;
    c->prof_bytes[cls] += bytes;
    if (c->prof_mask & (1u << cls)) {
      a = next_event(c);
      b = next_event(c);
      cudaEventRecord(a, c->stream);
    }
  }
  ~Prof() {
    if (b) {
      cudaEventRecord(b, c->stream);
      c->prof_recs.push_back({cls, a, b});
    }
  }
};
}  // namespace

namespace {

constexpr int PREFILL_CHUNK = 512;
// The residual pass of spec_verify keeps one sum per vocabulary chunk of
// 8192 logits in shared memory (64 slots).
constexpr int MAX_VOCAB = 64 * 8192;

int fail(uno_ctx* c, int code, const std::string& msg) {
  if (c) c->err = msg;
  return code;
}

#define CK(call)                                                                            \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess)                                                                  \
      return fail(c, UNO_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_));     \
  } while (0)

template <typename P>
cudaError_t dalloc(P** p, size_t bytes) {
  return cudaMalloc((void**)p, bytes ? bytes : 16);
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// ---------------------------------------------------------------------------
// GEMM dispatch.
// ---------------------------------------------------------------------------
struct Gemm {
  GemmParams p{};
  Gemm(const void* X, int ldx, int M, int K) {
    p.X = X; p.ldx = ldx; p.M = M; p.K = K; p.N = 0; p.nseg = 0; p.U = nullptr; p.r = 0;
    p.alpha = 1.f; p.row_gate = nullptr;
  }
  Gemm& seg(const void* W, int n, const void* lB = nullptr, int u_off = 0) {
    p.seg[p.nseg] = GemmSeg{W, lB, p.N, n, u_off};
    p.nseg++;
    p.N += n;
    return *this;
  }
  Gemm& lora(const void* U, int ldu, int r) { p.U = U; p.ldu = ldu; p.r = r; return *this; }
  Gemm& epi(int e, void* out, int ldo, float alpha = 1.f, const float* gate = nullptr) {
    p.epi = e; p.out = out; p.ldo = ldo; p.alpha = alpha; p.row_gate = gate;
    return *this;
  }
};

// Algorithmic bytes of one GEMM launch: weights, LoRA-B, activations and U
// read once, outputs written once (read too for the residual add).
double gemm_bytes(const GemmParams& p, size_t esz) {
  double b = (double)esz * ((double)p.N * p.K + (double)p.M * p.K);
  if (p.U) b += (double)esz * ((double)p.N * p.r + (double)p.M * p.r);
  const double out = (double)p.M * p.N;
  if (p.epi == EPI_STORE || p.epi == EPI_GATED) b += out * esz;
  else if (p.epi == EPI_STORE_F32) b += out * 4;
  else b += out * 8;
  return b;
}

template <typename T>
void launch_gemm(uno_ctx* c, const Gemm& g, cudaStream_t st) {
  const GemmParams& p = g.p;
  if (p.M <= 0 || p.N <= 0) return;
  Prof prof(c, UNO_K_GEMM, gemm_bytes(p, sizeof(T)));
  const dim3 block(256);
  if (p.M <= 8) {
    gemm_simt_kernel<T, 8, 4><<<dim3(ceil_div(p.N, 32), ceil_div(p.M, 8)), block, 0, st>>>(p);
  } else if (p.M <= 16) {
    gemm_simt_kernel<T, 16, 4><<<dim3(ceil_div(p.N, 32), ceil_div(p.M, 16)), block, 0, st>>>(p);
  } else {
    gemm_simt_kernel<T, 32, 2><<<dim3(ceil_div(p.N, 16), ceil_div(p.M, 32)), block, 0, st>>>(p);
  }
}

// ---------------------------------------------------------------------------
// Attention dispatch.
// ---------------------------------------------------------------------------
template <typename T, int HD>
int launch_attn_hd(uno_ctx* c, AttnParams& p, int n_req, cudaStream_t st) {
  const size_t smem = (size_t)(ATT_MAXQ * HD + ATT_KT * (HD + 1) + ATT_KT * HD) * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    CK(cudaFuncSetAttribute(attn_simt_kernel<T, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                            (int)smem));
    attr_set = true;
  }
  const dim3 grid(p.n_splits, p.n_qtiles, n_req * p.Hkv);
  Prof prof(c, UNO_K_ATTN, 0.0);
  attn_simt_kernel<T, HD><<<grid, ATT_THREADS, smem, st>>>(p);
  return UNO_OK;
}

template <typename T>
int launch_attn(uno_ctx* c, int layer, int n_req, int rows_per_req, bool decode) {
  const uno_shape& s = c->s;
  AttnParams p{};
  p.qkv = c->qkv;
  p.ld_qkv = (s.n_heads + 2 * s.n_kv_heads) * s.head_dim;
  p.out = c->attn;
  p.ld_out = s.n_heads * s.head_dim;
  p.kv = c->kv;
  p.layer = layer;
  p.H = s.n_heads;
  p.Hkv = s.n_kv_heads;
  p.scale = 1.0f / sqrtf((float)s.head_dim);
  p.rows_per_req = rows_per_req;
  p.row_pos = c->row_pos;
  p.row_slot = c->row_slot;
  const int G = s.n_heads / s.n_kv_heads;
  const int TQ = ATT_MAXQ / G;
  p.n_qtiles = ceil_div(rows_per_req, TQ);
  const int groups = n_req * s.n_kv_heads * p.n_qtiles;
  int S = 1;
  if (decode) {
    S = ceil_div(2 * 148, groups);
    const int max_tiles = ceil_div(c->max_ctx + c->B + 2, ATT_KT);
    S = std::max(1, std::min(S, max_tiles / 8));
    while (S > 1 && (size_t)groups * S * ATT_MAXQ * (s.head_dim + 2) > c->att_ws_floats) --S;
    if (groups > c->att_groups_max) S = 1;
  }
  p.n_splits = S;
  p.ws = c->att_ws;
  p.counters = c->att_counters;
  switch (s.head_dim) {
    case 16: return launch_attn_hd<T, 16>(c, p, n_req, c->stream);
    case 32: return launch_attn_hd<T, 32>(c, p, n_req, c->stream);
    case 64: return launch_attn_hd<T, 64>(c, p, n_req, c->stream);
    case 128: return launch_attn_hd<T, 128>(c, p, n_req, c->stream);
    default: return fail(c, UNO_ERR_UNSUPPORTED, "head_dim must be 16, 32, 64 or 128");
  }
}

// ---------------------------------------------------------------------------
// One forward pass over M = n_req * rows_per_req rows.
// ---------------------------------------------------------------------------
template <typename T>
int forward(uno_ctx* c, int kind, int n_req, int rows_per_req, const int32_t* req_ids,
            const int32_t* prompt, int prefill_slot, int prefill_pos0, float* logits) {
  const uno_shape& s = c->s;
  const int M = n_req * rows_per_req;
  const int d = s.d_model, H = s.n_heads, Hkv = s.n_kv_heads, hd = s.head_dim, F = s.ffn_dim;
  const int r = c->r;
  const int qkv_ld = (H + 2 * Hkv) * hd;
  const bool lora = (kind == PASS_DRAFT);
  cudaStream_t st = c->stream;

  RowArgs ra{};
  ra.kind = kind;
  ra.rows_per_req = rows_per_req;
  ra.req_slot = req_ids;
  ra.cached = c->d_cached;
  ra.pending = c->d_pending;
  ra.drafts = c->drafts;
  ra.B = c->B;
  ra.prompt = prompt;
  ra.prefill_slot = prefill_slot;
  ra.mask_id = s.mask_id;
  ra.vocab = s.vocab;
  ra.max_batch = c->max_batch;
  ra.lora_scale = c->lscale;
  ra.row_pos = c->row_pos;
  ra.row_slot = c->row_slot;
  ra.row_gate = c->row_gate;
  ra.embed = c->embed;
  ra.d = d;
  ra.x = c->x;
  ra.status = c->d_status;
  ra.prefill_pos0 = prefill_pos0;
  {
    Prof prof(c, UNO_K_OTHER, 0.0);
    build_rows_kernel<T><<<M, 256, 0, st>>>(ra);
  }
  auto other = [&](auto launch) {
    Prof prof(c, UNO_K_OTHER, 0.0);
    launch();
  };

  const int xn_ld = std::max(d, F);
  const int ldu = 3 * r;
  for (int l = 0; l < s.n_layers; ++l) {
    other([&] {
      rmsnorm_kernel<T, 256><<<M, 256, 0, st>>>(c->x, (const T*)c->attn_norm[l], (T*)c->xn, d,
                                               xn_ld, s.rms_eps);
    });
    if (lora) {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->lA[UNO_PROJ_Q][l], r).seg(c->lA[UNO_PROJ_K][l], r).seg(c->lA[UNO_PROJ_V][l], r);
      g.epi(EPI_GATED, c->U, ldu, 1.f, c->row_gate);
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->w[UNO_PROJ_Q][l], H * hd, lora ? c->lB[UNO_PROJ_Q][l] : nullptr, 0)
          .seg(c->w[UNO_PROJ_K][l], Hkv * hd, lora ? c->lB[UNO_PROJ_K][l] : nullptr, r)
          .seg(c->w[UNO_PROJ_V][l], Hkv * hd, lora ? c->lB[UNO_PROJ_V][l] : nullptr, 2 * r);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_STORE, c->qkv, qkv_ld);
      launch_gemm<T>(c, g, st);
    }
    other([&] {
      rope_kv_kernel<T><<<M, 128, 0, st>>>((T*)c->qkv, qkv_ld, c->row_pos, c->row_slot, c->cos_t,
                                           c->sin_t, c->max_pos, H, Hkv, hd, c->kv, l, c->d_status);
    });
    {
      const int rc = launch_attn<T>(c, l, n_req, rows_per_req, kind != PASS_PREFILL);
      if (rc) return rc;
    }
    if (lora) {
      Gemm g(c->attn, H * hd, M, H * hd);
      g.seg(c->lA[UNO_PROJ_O][l], r).epi(EPI_GATED, c->U, ldu, 1.f, c->row_gate);
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->attn, H * hd, M, H * hd);
      g.seg(c->w[UNO_PROJ_O][l], d, lora ? c->lB[UNO_PROJ_O][l] : nullptr, 0);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_ADD_F32, c->x, d);
      launch_gemm<T>(c, g, st);
    }
    other([&] {
      rmsnorm_kernel<T, 256><<<M, 256, 0, st>>>(c->x, (const T*)c->ffn_norm[l], (T*)c->xn, d,
                                               xn_ld, s.rms_eps);
    });
    if (lora) {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->lA[UNO_PROJ_GATE][l], r).seg(c->lA[UNO_PROJ_UP][l], r);
      g.epi(EPI_GATED, c->U, ldu, 1.f, c->row_gate);
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->w[UNO_PROJ_GATE][l], F, lora ? c->lB[UNO_PROJ_GATE][l] : nullptr, 0)
          .seg(c->w[UNO_PROJ_UP][l], F, lora ? c->lB[UNO_PROJ_UP][l] : nullptr, r);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_STORE, c->gu, 2 * F);
      launch_gemm<T>(c, g, st);
    }
    other([&] { swiglu_kernel<T><<<M, 256, 0, st>>>((const T*)c->gu, F, (T*)c->xn); });
    if (lora) {
      Gemm g(c->xn, F, M, F);
      g.seg(c->lA[UNO_PROJ_DOWN][l], r).epi(EPI_GATED, c->U, ldu, 1.f, c->row_gate);
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->xn, F, M, F);
      g.seg(c->w[UNO_PROJ_DOWN][l], d, lora ? c->lB[UNO_PROJ_DOWN][l] : nullptr, 0);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_ADD_F32, c->x, d);
      launch_gemm<T>(c, g, st);
    }
  }
  if (logits) {
    other([&] {
      rmsnorm_kernel<T, 256><<<M, 256, 0, st>>>(c->x, (const T*)c->final_norm, (T*)c->xn, d,
                                               xn_ld, s.rms_eps);
    });
    Gemm g(c->xn, xn_ld, M, d);
    g.seg(c->lm_head, s.vocab).epi(EPI_STORE_F32, logits, s.vocab, 1.0f / s.temperature);
    launch_gemm<T>(c, g, st);
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

int forward_any(uno_ctx* c, int kind, int n_req, int rows_per_req, const int32_t* req_ids,
                const int32_t* prompt, int prefill_slot, int prefill_pos0, float* logits) {
  if (c->s.dtype == UNO_BF16)
    return forward<bf16>(c, kind, n_req, rows_per_req, req_ids, prompt, prefill_slot, prefill_pos0,
                         logits);
  return forward<float>(c, kind, n_req, rows_per_req, req_ids, prompt, prefill_slot, prefill_pos0,
                        logits);
}

void chunking(int V, int* ch, int* nch) {
  int c = V < 8192 ? ((V + 3) / 4) * 4 : 8192;
  *ch = c;
  *nch = (V + c - 1) / c;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* uno_last_error(const uno_ctx* ctx) { return ctx ? ctx->err.c_str() : "null context"; }

int uno_init(const uno_shape* shape, const uno_weights* wts, int lora_rank, float lora_alpha,
             int block_B, int max_batch, int max_ctx, uint64_t seed, uno_stream_t stream,
             uno_ctx** out) {
  if (!shape || !wts || !out) return UNO_ERR_ARG;
  *out = nullptr;
  const uno_shape& s = *shape;
  if (s.n_layers < 1 || s.d_model < 1 || s.n_heads < 1 || s.n_kv_heads < 1 ||
      s.n_heads % s.n_kv_heads || s.head_dim < 2 || s.ffn_dim < 1 || s.vocab < 2 ||
      s.mask_id < 0 || s.mask_id >= s.vocab || lora_rank < 1 || block_B < 2 || block_B > 64 ||
      max_batch < 1 || max_ctx < 2 || !(s.temperature > 0.f) ||
      (s.dtype != UNO_F32 && s.dtype != UNO_BF16))
    return UNO_ERR_ARG;
  const int G = s.n_heads / s.n_kv_heads;
  const int vec = s.dtype == UNO_BF16 ? 8 : 4;
  if (G > ATT_MAXQ || s.vocab % 4 || s.vocab > MAX_VOCAB || s.d_model % vec || s.ffn_dim % vec ||
      lora_rank % vec ||
      (s.n_heads * s.head_dim) % vec ||
      (s.head_dim != 16 && s.head_dim != 32 && s.head_dim != 64 && s.head_dim != 128))
    return UNO_ERR_UNSUPPORTED;
  if (!wts->embed || !wts->lm_head || !wts->final_norm || !wts->attn_norm || !wts->ffn_norm)
    return UNO_ERR_ARG;
  for (int p = 0; p < UNO_N_PROJ; ++p)
    if (!wts->w[p] || !wts->lora_A[p] || !wts->lora_B[p]) return UNO_ERR_ARG;

  uno_ctx* c = new uno_ctx();
  c->s = s;
  c->r = lora_rank;
  c->alpha = lora_alpha;
  c->lscale = lora_alpha / (float)lora_rank;
  c->B = block_B;
  c->max_batch = max_batch;
  c->max_ctx = max_ctx;
  c->seed = seed;
  c->stream = (cudaStream_t)stream;
  c->esz = s.dtype == UNO_BF16 ? 2 : 4;
  c->embed = wts->embed;
  c->lm_head = wts->lm_head;
  c->final_norm = wts->final_norm;
  const int L = s.n_layers;
  c->attn_norm.assign(wts->attn_norm, wts->attn_norm + L);
  c->ffn_norm.assign(wts->ffn_norm, wts->ffn_norm + L);
  for (int p = 0; p < UNO_N_PROJ; ++p) {
    c->w[p].assign(wts->w[p], wts->w[p] + L);
    c->lA[p].assign(wts->lora_A[p], wts->lora_A[p] + L);
    c->lB[p].assign(wts->lora_B[p], wts->lora_B[p] + L);
    for (int l = 0; l < L; ++l)
      if (!c->w[p][l] || !c->lA[p][l] || !c->lB[p][l]) {
        delete c;
        return UNO_ERR_ARG;
      }
  }

  auto oom = [&](const char* what) {
    std::string m = std::string("allocation failed: ") + what;
    uno_destroy(c);
    (void)m;
    return UNO_ERR_OOM;
  };
  const int H = s.n_heads, Hkv = s.n_kv_heads, hd = s.head_dim, d = s.d_model, F = s.ffn_dim;
  const int V = s.vocab, B = block_B;

  // KV pool
  const int ppr = ceil_div(max_ctx + B + 2, KV_PAGE);
  const int n_pages = max_batch * ppr;
  const size_t kv_bytes = (size_t)L * n_pages * 2 * Hkv * KV_PAGE * hd * c->esz;
  if (dalloc(&c->kv_pool, kv_bytes) != cudaSuccess) return oom("kv pool");
  if (dalloc(&c->d_page_table, (size_t)max_batch * ppr * 4) != cudaSuccess) return oom("pages");
  if (dalloc(&c->d_cached, (size_t)max_batch * 4) != cudaSuccess) return oom("state");
  if (dalloc(&c->d_pending, (size_t)max_batch * 4) != cudaSuccess) return oom("state");
  if (dalloc(&c->d_stream, (size_t)max_batch * 4) != cudaSuccess) return oom("state");
  c->kv = KvLayout{c->kv_pool, n_pages, Hkv, hd, ppr, c->d_page_table};
  c->free_pages.resize(n_pages);
  for (int i = 0; i < n_pages; ++i) c->free_pages[i] = n_pages - 1 - i;
  c->slot_used.assign(max_batch, 0);
  c->h_page_table.assign((size_t)max_batch * ppr, 0);
  cudaMemset(c->d_page_table, 0, (size_t)max_batch * ppr * 4);
  cudaMemset(c->d_cached, 0, (size_t)max_batch * 4);
  cudaMemset(c->d_pending, 0, (size_t)max_batch * 4);
  cudaMemset(c->d_stream, 0, (size_t)max_batch * 4);

  // activations
  const int M = std::max(max_batch * (B + 1), PREFILL_CHUNK);
  c->M_max = M;
  const size_t e = c->esz;
  if (dalloc(&c->x, (size_t)M * d * 4) != cudaSuccess) return oom("x");
  if (dalloc(&c->xn, (size_t)M * std::max(d, F) * e) != cudaSuccess) return oom("xn");
  if (dalloc(&c->qkv, (size_t)M * (H + 2 * Hkv) * hd * e) != cudaSuccess) return oom("qkv");
  if (dalloc(&c->attn, (size_t)M * H * hd * e) != cudaSuccess) return oom("attn");
  if (dalloc(&c->gu, (size_t)M * 2 * F * e) != cudaSuccess) return oom("gu");
  if (dalloc(&c->U, (size_t)M * 3 * lora_rank * e) != cudaSuccess) return oom("U");
  if (dalloc(&c->row_pos, (size_t)M * 4) != cudaSuccess) return oom("rows");
  if (dalloc(&c->row_slot, (size_t)M * 4) != cudaSuccess) return oom("rows");
  if (dalloc(&c->row_gate, (size_t)M * 4) != cudaSuccess) return oom("rows");

  // RoPE table, double precision on the host
  c->max_pos = ppr * KV_PAGE;
  {
    const int half = hd / 2;
    std::vector<float> ct((size_t)c->max_pos * half), stb((size_t)c->max_pos * half);
    for (int pos = 0; pos < c->max_pos; ++pos)
      for (int i = 0; i < half; ++i) {
        const double inv = std::pow((double)s.rope_theta, -2.0 * i / hd);
        const double a = (double)pos * inv;
        ct[(size_t)pos * half + i] = (float)std::cos(a);
        stb[(size_t)pos * half + i] = (float)std::sin(a);
      }
    if (dalloc(&c->cos_t, ct.size() * 4) != cudaSuccess) return oom("rope");
    if (dalloc(&c->sin_t, ct.size() * 4) != cudaSuccess) return oom("rope");
    cudaMemcpy(c->cos_t, ct.data(), ct.size() * 4, cudaMemcpyHostToDevice);
    cudaMemcpy(c->sin_t, stb.data(), stb.size() * 4, cudaMemcpyHostToDevice);
  }

  // logits and sampler workspaces
  chunking(V, &c->ch, &c->nch);
  if (dalloc(&c->logits_d, (size_t)max_batch * (B + 1) * V * 4) != cudaSuccess) return oom("logits");
  if (dalloc(&c->logits_v, (size_t)max_batch * B * V * 4) != cudaSuccess) return oom("logits");
  if (dalloc(&c->drafts, (size_t)max_batch * B * 4) != cudaSuccess) return oom("drafts");
  if (dalloc(&c->lse_q, (size_t)max_batch * B * 4) != cudaSuccess) return oom("lse");
  const size_t rows_ws = (size_t)max_batch * 2 * B;
  if (dalloc(&c->partial, rows_ws * c->nch * sizeof(float2)) != cudaSuccess) return oom("partial");
  if (dalloc(&c->lse_ws, rows_ws * 4) != cudaSuccess) return oom("lse");
  if (dalloc(&c->row_counter, rows_ws * 4) != cudaSuccess) return oom("counters");
  if (dalloc(&c->req_counter, (size_t)max_batch * 4) != cudaSuccess) return oom("counters");
  cudaMemset(c->row_counter, 0, rows_ws * 4);
  cudaMemset(c->req_counter, 0, (size_t)max_batch * 4);
  cudaMemset(c->drafts, 0, (size_t)max_batch * B * 4);

  // attention split workspace: up to 2 waves of 148 CTAs
  c->att_groups_max = max_batch * Hkv * ceil_div(B + 1, ATT_MAXQ / (H / Hkv));
  c->att_ws_floats = (size_t)std::max(c->att_groups_max, 2 * 148 + c->att_groups_max) * ATT_MAXQ * (hd + 2);
  if (dalloc(&c->att_ws, c->att_ws_floats * 4) != cudaSuccess) return oom("attention ws");
  if (dalloc(&c->att_counters, (size_t)c->att_groups_max * 4) != cudaSuccess) return oom("attention ws");
  cudaMemset(c->att_counters, 0, (size_t)c->att_groups_max * 4);
  if (dalloc(&c->d_status, 4) != cudaSuccess) return oom("status");
  cudaMemset(c->d_status, 0, 4);
  if (cudaDeviceSynchronize() != cudaSuccess) {
    uno_destroy(c);
    return UNO_ERR_CUDA;
  }
  *out = c;
  return UNO_OK;
}

int uno_destroy(uno_ctx* c) {
  if (!c) return UNO_ERR_ARG;
  if (c->stream) cudaStreamSynchronize(c->stream);
  cudaDeviceSynchronize();
  void* bufs[] = {c->kv_pool, c->d_page_table, c->d_cached, c->d_pending, c->d_stream, c->x,
                  c->xn, c->qkv, c->attn, c->gu, c->U, c->row_pos, c->row_slot, c->row_gate,
                  c->cos_t, c->sin_t, c->logits_d, c->logits_v, c->drafts, c->lse_q, c->partial,
                  c->lse_ws, c->row_counter, c->req_counter, c->att_ws, c->att_counters,
                  c->d_status};
  for (void* b : bufs)
    if (b) cudaFree(b);
  for (cudaEvent_t e : c->ev_pool) cudaEventDestroy(e);
  delete c;
  return UNO_OK;
}

int uno_prefill(uno_ctx* c, int n_req, const int32_t* prompts_dev, int prompt_stride,
                const int32_t* prompt_lens_host, const uint32_t* streams_host,
                int32_t* req_ids_host_out) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_req < 1 || !prompts_dev || !prompt_lens_host || !req_ids_host_out || prompt_stride < 1)
    return fail(c, UNO_ERR_ARG, "bad prefill arguments");
  int free_slots = 0;
  for (int u : c->slot_used) free_slots += !u;
  const int ppr = c->kv.pages_per_req;
  if (free_slots < n_req || (int)c->free_pages.size() < n_req * ppr)
    return fail(c, UNO_ERR_CAPACITY, "no free request slot or KV pages");
  for (int i = 0; i < n_req; ++i)
    if (prompt_lens_host[i] < 1 || prompt_lens_host[i] > c->max_ctx || prompt_lens_host[i] > prompt_stride)
      return fail(c, UNO_ERR_ARG, "prompt length out of range");
  for (int i = 0; i < n_req; ++i) {
    int slot = 0;
    while (c->slot_used[slot]) ++slot;
    c->slot_used[slot] = 1;
    for (int pi = 0; pi < ppr; ++pi) {
      c->h_page_table[(size_t)slot * ppr + pi] = c->free_pages.back();
      c->free_pages.pop_back();
    }
    CK(cudaMemcpyAsync(c->d_page_table + (size_t)slot * ppr, c->h_page_table.data() + (size_t)slot * ppr,
                       ppr * 4, cudaMemcpyHostToDevice, c->stream));
    const uint32_t sid = streams_host ? streams_host[i] : (uint32_t)slot;
    CK(cudaMemcpyAsync(c->d_stream + slot, &sid, 4, cudaMemcpyHostToDevice, c->stream));
    CK(cudaStreamSynchronize(c->stream));  // host staging values above are locals
    req_ids_host_out[i] = slot;
    const int P = prompt_lens_host[i];
    const int32_t* prompt = prompts_dev + (size_t)i * prompt_stride;
    for (int p0 = 0; p0 < P - 1; p0 += PREFILL_CHUNK) {
      const int n = std::min(PREFILL_CHUNK, P - 1 - p0);
      const int rc = forward_any(c, PASS_PREFILL, 1, n, nullptr, prompt + p0, slot, p0, nullptr);
      if (rc) return rc;
    }
    init_slot_kernel<<<1, 1, 0, c->stream>>>(prompt, P, slot, c->d_cached, c->d_pending);
    CK(cudaGetLastError());
  }
  return UNO_OK;
}

int uno_spec_step(uno_ctx* c, int n_req, const int32_t* req_ids_dev, int32_t* out_tokens_dev,
                  int32_t* n_new_dev) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_req < 1 || n_req > c->max_batch || !req_ids_dev || !out_tokens_dev || !n_new_dev)
    return fail(c, UNO_ERR_ARG, "bad spec_step arguments");
  const int B = c->B, V = c->s.vocab;
  c->last_n_req = n_req;
  int rc = forward_any(c, PASS_DRAFT, n_req, B + 1, req_ids_dev, nullptr, 0, 0, c->logits_d);
  if (rc) return rc;
  {
    SampleArgs a{};
    a.logits = c->logits_d;
    a.V = V; a.nch = c->nch; a.ch = c->ch;
    a.rows_per_req = B;
    a.logit_rows_per_req = B + 1;
    a.ar_mode = 0;
    a.req_slot = req_ids_dev;
    a.cached = c->d_cached;
    a.pending = c->d_pending;
    a.slot_stream = c->d_stream;
    a.seed = c->seed;
    a.out_tok = c->drafts;
    a.out_stride = B;
    a.lse_out = c->lse_q;
    a.partial = c->partial;
    a.row_counter = c->row_counter;
    a.status = c->d_status;
    Prof prof(c, UNO_K_SAMPLE, (double)n_req * B * V * 4);
    sample_rows_kernel<<<dim3(c->nch, n_req * B), SAMPLE_THREADS, 0, c->stream>>>(a);
  }
  rc = forward_any(c, PASS_VERIFY, n_req, B, req_ids_dev, nullptr, 0, 0, c->logits_v);
  if (rc) return rc;
  {
    VerifyArgs a{};
    a.p = c->logits_v;
    a.q = c->logits_d;
    a.V = V; a.nch = c->nch; a.ch = c->ch;
    a.n_tests = B - 1;
    a.p_req_rows = B;
    a.q_req_rows = B + 1;
    a.p_row0 = 0;
    a.q_row0 = 2;
    a.bonus_row = B - 1;
    a.drafts = c->drafts; a.drafts_stride = B; a.drafts_off = 1;
    a.lse_q_in = c->lse_q; a.lse_q_stride = B; a.lse_q_off = 1;
    a.seed = c->seed;
    a.req_slot = req_ids_dev;
    a.cached = c->d_cached;
    a.pending = c->d_pending;
    a.slot_stream = c->d_stream;
    a.first_tok = c->drafts;
    a.out_tok = out_tokens_dev;
    a.out_stride = B + 1;
    a.n_out = n_new_dev;
    a.partial = c->partial;
    a.lse = c->lse_ws;
    a.row_counter = c->row_counter;
    a.req_counter = c->req_counter;
    a.rows_red = B;      // B - 1 test rows + the bonus row; lse of q comes from draft_sample
    a.n_p = B;
    a.status = c->d_status;
    Prof prof(c, UNO_K_VERIFY, (double)n_req * B * V * 4);
    spec_verify_kernel<<<dim3(c->nch, n_req * B), SAMPLE_THREADS, 0, c->stream>>>(a);
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

int uno_ar_step(uno_ctx* c, int n_req, const int32_t* req_ids_dev, int32_t* out_tokens_dev) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_req < 1 || n_req > c->max_batch || !req_ids_dev || !out_tokens_dev)
    return fail(c, UNO_ERR_ARG, "bad ar_step arguments");
  c->last_n_req = n_req;
  int rc = forward_any(c, PASS_AR, n_req, 1, req_ids_dev, nullptr, 0, 0, c->logits_d);
  if (rc) return rc;
  SampleArgs a{};
  a.logits = c->logits_d;
  a.V = c->s.vocab; a.nch = c->nch; a.ch = c->ch;
  a.rows_per_req = 1;
  a.logit_rows_per_req = 1;
  a.ar_mode = 1;
  a.req_slot = req_ids_dev;
  a.cached = c->d_cached;
  a.pending = c->d_pending;
  a.slot_stream = c->d_stream;
  a.seed = c->seed;
  a.out_tok = out_tokens_dev;
  a.out_stride = 1;
  a.partial = c->partial;
  a.row_counter = c->row_counter;
  a.status = c->d_status;
  {
    Prof prof(c, UNO_K_SAMPLE, (double)n_req * a.V * 4);
    sample_rows_kernel<<<dim3(c->nch, n_req), SAMPLE_THREADS, 0, c->stream>>>(a);
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

int uno_profile_begin(uno_ctx* c, unsigned mask) {
  if (!c) return UNO_ERR_ARG;
  CK(cudaStreamSynchronize(c->stream));
  c->prof_mask = mask;
  c->prof_recs.clear();
  c->ev_next = 0;
  for (int k = 0; k < UNO_K_N; ++k) {
    c->prof_launches[k] = 0;
    c->prof_bytes[k] = 0.0;
  }
  return UNO_OK;
}

int uno_profile_end(uno_ctx* c, int64_t* launches, double* ms, double* bytes) {
  if (!c) return UNO_ERR_ARG;
  CK(cudaStreamSynchronize(c->stream));
  double t[UNO_K_N] = {};
  for (const auto& r : c->prof_recs) {
    float e = 0.f;
    CK(cudaEventElapsedTime(&e, r.a, r.b));
    t[r.cls] += e;
  }
  for (int k = 0; k < UNO_K_N; ++k) {
    if (launches) launches[k] = c->prof_launches[k];
    if (ms) ms[k] = t[k];
    if (bytes) bytes[k] = c->prof_bytes[k];
  }
  c->prof_mask = 0;
  c->prof_recs.clear();
  c->ev_next = 0;
  return UNO_OK;
}

int uno_release(uno_ctx* c, int req) {
  if (!c) return UNO_ERR_ARG;
  if (req < 0 || req >= c->max_batch || !c->slot_used[req]) return fail(c, UNO_ERR_ARG, "unknown request id");
  CK(cudaStreamSynchronize(c->stream));
  const int ppr = c->kv.pages_per_req;
  for (int pi = 0; pi < ppr; ++pi) c->free_pages.push_back(c->h_page_table[(size_t)req * ppr + pi]);
  c->slot_used[req] = 0;
  return UNO_OK;
}

int uno_status(uno_ctx* c) {
  if (!c) return UNO_ERR_ARG;
  CK(cudaStreamSynchronize(c->stream));
  int32_t st = 0;
  CK(cudaMemcpy(&st, c->d_status, 4, cudaMemcpyDeviceToHost));
  if (st) {
    CK(cudaMemset(c->d_status, 0, 4));
    return fail(c, UNO_ERR_DEVICE_CHECK, "device check flag " + std::to_string(st));
  }
  return UNO_OK;
}

int uno_request_state(uno_ctx* c, int req, int32_t* cached_out, int32_t* pending_out) {
  if (!c || !cached_out || !pending_out) return UNO_ERR_ARG;
  if (req < 0 || req >= c->max_batch || !c->slot_used[req]) return fail(c, UNO_ERR_ARG, "unknown request id");
  CK(cudaStreamSynchronize(c->stream));
  CK(cudaMemcpy(cached_out, c->d_cached + req, 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(pending_out, c->d_pending + req, 4, cudaMemcpyDeviceToHost));
  return UNO_OK;
}

int uno_debug_read(uno_ctx* c, int which, void* dst, size_t bytes) {
  if (!c || !dst) return UNO_ERR_ARG;
  const size_t V = c->s.vocab, B = c->B, mb = c->max_batch;
  const void* src = nullptr;
  size_t cap = 0;
  switch (which) {
    case UNO_DBG_LOGITS_DRAFT: src = c->logits_d; cap = mb * (B + 1) * V * 4; break;
    case UNO_DBG_LOGITS_VERIFY: src = c->logits_v; cap = mb * B * V * 4; break;
    case UNO_DBG_DRAFTS: src = c->drafts; cap = mb * B * 4; break;
    case UNO_DBG_LOGITS_AR: src = c->logits_d; cap = mb * V * 4; break;
    default: return fail(c, UNO_ERR_ARG, "unknown debug buffer");
  }
  if (bytes > cap) return fail(c, UNO_ERR_ARG, "debug read larger than the buffer");
  CK(cudaStreamSynchronize(c->stream));
  CK(cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost));
  return UNO_OK;
}

int uno_debug_kv(uno_ctx* c, int req, int layer, int pos0, int n, void* k_host, void* v_host) {
  if (!c || !k_host || !v_host) return UNO_ERR_ARG;
  if (req < 0 || req >= c->max_batch || !c->slot_used[req] || layer < 0 ||
      layer >= c->s.n_layers || pos0 < 0 || n < 0 || pos0 + n > c->max_pos)
    return fail(c, UNO_ERR_ARG, "bad debug_kv arguments");
  CK(cudaStreamSynchronize(c->stream));
  const int Hkv = c->s.n_kv_heads, hd = c->s.head_dim, ppr = c->kv.pages_per_req;
  const size_t row = (size_t)hd * c->esz;
  for (int i = 0; i < n; ++i) {
    const int pos = pos0 + i;
    const int page = c->h_page_table[(size_t)req * ppr + pos / KV_PAGE];
    for (int h = 0; h < Hkv; ++h)
      for (int kv = 0; kv < 2; ++kv) {
        const size_t off = ((((size_t)layer * c->kv.n_pages + page) * 2 + kv) * Hkv + h) * KV_PAGE * hd +
                           (size_t)(pos % KV_PAGE) * hd;
        char* dst = (char*)(kv ? v_host : k_host) + ((size_t)i * Hkv + h) * row;
        CK(cudaMemcpy(dst, (char*)c->kv_pool + off * c->esz, row, cudaMemcpyDeviceToHost));
      }
  }
  return UNO_OK;
}

// ---------------------------------------------------------------------------
// Stand-alone spec_verify.
// ---------------------------------------------------------------------------
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct VerifyWs {
  size_t counters, req_counters, lse, partial, total;
};
static VerifyWs verify_ws_layout(int n_req, int n_tests, int vocab) {
  int ch, nch;
  chunking(vocab, &ch, &nch);
  const size_t rows = (size_t)n_req * 2 * n_tests;
  VerifyWs w{};
  w.counters = 0;
  w.req_counters = align256(rows * 4);
  w.lse = w.req_counters + align256((size_t)n_req * 4);
  w.partial = w.lse + align256(rows * 4);
  w.total = w.partial + align256(rows * nch * sizeof(float2));
  return w;
}

size_t uno_spec_verify_workspace_bytes(int n_req, int n_tests, int vocab) {
  if (n_req < 1 || n_tests < 1 || vocab < 4) return 0;
  return verify_ws_layout(n_req, n_tests, vocab).total;
}

int uno_spec_verify(const float* p, const float* q, const int32_t* drafts, int n_req, int n_tests,
                    int vocab, uint64_t seed, const uint32_t* streams, const int32_t* pos0,
                    int32_t* out_tokens, int32_t* n_out, void* ws, size_t ws_bytes,
                    uno_stream_t stream) {
  if (!p || !q || !drafts || !streams || !pos0 || !out_tokens || !n_out || !ws) return UNO_ERR_ARG;
  if (n_req < 1 || n_tests < 1 || vocab < 4 || vocab % 4 || vocab > MAX_VOCAB || n_tests > 1024)
    return UNO_ERR_ARG;
  const VerifyWs w = verify_ws_layout(n_req, n_tests, vocab);
  if (ws_bytes < w.total || ((uintptr_t)ws & 255)) return UNO_ERR_ARG;
  int ch, nch;
  chunking(vocab, &ch, &nch);
  if ((long long)n_req * 2 * n_tests > 65535LL) return UNO_ERR_ARG;
  VerifyArgs a{};
  a.p = p; a.q = q;
  a.V = vocab; a.nch = nch; a.ch = ch;
  a.n_tests = n_tests;
  a.p_req_rows = n_tests; a.q_req_rows = n_tests;
  a.p_row0 = 0; a.q_row0 = 0;
  a.bonus_row = -1;
  a.drafts = drafts; a.drafts_stride = n_tests; a.drafts_off = 0;
  a.lse_q_in = nullptr;
  a.seed = seed;
  a.req_slot = nullptr;
  a.streams = streams; a.pos0 = pos0;
  a.out_tok = out_tokens; a.out_stride = n_tests + 1; a.n_out = n_out;
  char* base = (char*)ws;
  a.row_counter = (unsigned*)(base + w.counters);
  a.req_counter = (unsigned*)(base + w.req_counters);
  a.lse = (float*)(base + w.lse);
  a.partial = (float2*)(base + w.partial);
  a.rows_red = 2 * n_tests;
  a.n_p = n_tests;
  a.status = nullptr;
  const int rows = n_req * 2 * n_tests;
  spec_verify_kernel<<<dim3(nch, rows), SAMPLE_THREADS, 0, (cudaStream_t)stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

}  // extern "C"
