// Per-row layer kernels of the model forward: row assembly + embedding
// gather, RMSNorm, RoPE + paged KV write, SwiGLU.
//
// The forward is the frozen AR transformer plus a per-row gated LoRA
// (summary page "通过离散扩散实现 LLM 无损加速：扩散增强自回归模型", section
// 方法关键点; blog page "…Uno 的无损加速之路", section Diffusion Distillation：
// 一步蒸馏 + 块级扩散: the gate turns the adapter off at clean positions and on
// at noised ones).  The residual stream is fp32; GEMM inputs are in the
// model dtype.
#pragma once

#include "common.cuh"

namespace uno {

// Paged KV pool: [n_layers][n_pages][n_planes][n_kv_heads][PAGE][head_dim].
// Planes: fp32 models K, V; bf16 models K_hi, K_lo, V in fp16 (the keys as a
// hi/lo pair: their rounding is the largest term of the logit error left
// once q is a pair too).
constexpr int KV_PAGE = 64;

struct KvLayout {
  void* pool;
  int n_pages, n_kv_heads, head_dim, pages_per_req;
  const int32_t* page_table;   // [max_batch][pages_per_req]
  int n_planes;                // 2 (K, V) or 3 (K_hi, K_lo, V)
  __device__ __forceinline__ int v_plane() const { return n_planes - 1; }
  __device__ __forceinline__ size_t offset(int layer, int slot, int pos, int plane, int head,
                                           int& ok) const {
    return offset_in_page(layer, page_of(slot, pos, ok), pos, plane, head);
  }
  // page of (slot, pos); ok = 0 (page 0 returned) when pos is outside the slot's pages
  __device__ __forceinline__ int page_of(int slot, int pos, int& ok) const {
    const int pi = pos / KV_PAGE;
    ok = (pos >= 0 && pi < pages_per_req);
    return ok ? __ldcg(page_table + (size_t)slot * pages_per_req + pi) : 0;
  }
  __device__ __forceinline__ size_t offset_in_page(int layer, int page, int pos, int plane,
                                                   int head) const {
    return ((((size_t)layer * n_pages + page) * n_planes + plane) * n_kv_heads + head) * KV_PAGE *
               head_dim +
           (size_t)(pos % KV_PAGE) * head_dim;
  }
  // distance between planes of the same (page, head, position), in elements
  __device__ __forceinline__ size_t plane_stride() const {
    return (size_t)n_kv_heads * KV_PAGE * head_dim;
  }
};

// Pass kinds (a pass is one forward over a set of rows).
enum PassKind : int { PASS_PREFILL = 0, PASS_DRAFT = 1, PASS_VERIFY = 2, PASS_AR = 3, PASS_TRAIN = 4,
                      PASS_COHORT = 5, PASS_TREE = 6 };

// Tree sampler: at most this many drafted chains; the scratch slot of chain
// j of request slot r is max_batch + r TREE_MAX_K + j.
constexpr int TREE_MAX_K = 4;

// The keys each query row sees, by the block-causal rule (blog page "…Uno
// 的无损加速之路", section Diffusion Distillation：一步蒸馏 + 块级扩散: a clean
// query sees clean keys up to its own position; a query of a noised block
// sees the clean keys before its block and the keys of its own block up to
// its own position).  Keys live in the pool under a slot and a position, so a
// row's keys are two ranges:
//   clean range:  slot cslot[r], positions [0, lim) with lim = pos + 1, or the
//                 block start for a noised row of the training form;
//   noised range: (training form only, blk[r] >= 0) the row's own slot
//                 row_slot[r], positions [blk[r], pos + 1).
// With blk null every row is "causal by position" in its own slot: the
// decode passes, where the noised block's keys share the request's slot.
struct KeyTiles {
  int slot1, n1;      // clean range: slot, pages 0 .. n1-1
  int slot2, p2, n2;  // noised range: slot, pages p2 .. p2+n2-1 (n2 = 0: none)
  bool overflow;      // a range reached past the slot's pages (clipped)
};
struct RowKeys {
  const int32_t* cslot;   // [M] clean-range slot (null: row_slot)
  const int32_t* blk;     // [M] noised block start, -1 for a clean row (null: all clean)
  __device__ __forceinline__ void ranges(const int32_t* row_pos, int r, int& lim, int& lo2,
                                         int& hi2) const {
    const int pos = __ldcg(row_pos + r);
    const int b = blk ? __ldcg(blk + r) : -1;
    lim = b < 0 ? pos + 1 : b;
    lo2 = b < 0 ? 0 : b;
    hi2 = b < 0 ? 0 : pos + 1;
  }
  // The page lists of rows row0 .. row0 + ntok - 1 (one request): the union of
  // their ranges, in pages of `page` keys.
  __device__ __forceinline__ KeyTiles tiles(const int32_t* row_pos, const int32_t* row_slot,
                                            int row0, int ntok, int page, int pages_per_req) const {
    KeyTiles t{__ldcg((cslot ? cslot : row_slot) + row0), 0, -1, 0, 0, false};
    int lim1 = 0, lo2 = 0x7fffffff, hi2 = 0;
    if (!blk) {
      // causal by position: a request's rows are in position order, so the
      // last row reaches furthest (one load on the decode passes' path)
      lim1 = __ldcg(row_pos + row0 + ntok - 1) + 1;
      ntok = 0;
    }
    for (int k = 0; k < ntok; ++k) {
      int lim, l2, h2;
      ranges(row_pos, row0 + k, lim, l2, h2);
      lim1 = max(lim1, lim);
      if (h2 > l2) {
        lo2 = min(lo2, l2);
        hi2 = max(hi2, h2);
        t.slot2 = __ldcg(row_slot + row0 + k);
      }
    }
    t.n1 = (lim1 + page - 1) / page;
    if (t.n1 > pages_per_req) { t.n1 = pages_per_req; t.overflow = true; }
    if (hi2 > 0) {
      t.p2 = lo2 / page;
      int e = (hi2 + page - 1) / page;
      if (e > pages_per_req) { e = pages_per_req; t.overflow = true; }
      t.n2 = max(0, e - t.p2);
    }
    return t;
  }
};

struct RowArgs {
  int kind;
  int rows_per_req;
  const int32_t* req_slot;     // [n_req] slot ids (decode passes)
  const int32_t* cached;       // [max_batch]
  const int32_t* pending;      // [max_batch]
  const int32_t* drafts;       // [n_req, B] (verify pass)
  int B;
  const int32_t* prompt;       // prefill: this request's prompt (device)
  int prefill_slot, prefill_pos0;
  int mask_id, vocab, max_batch;
  float lora_scale;
  int32_t* row_pos; int32_t* row_slot; float* row_gate;   // outputs [M]
  const void* embed; int d;    // [vocab, d] model dtype
  float* x;                    // [M, d] fp32 residual
  int32_t* status;
  unsigned* zero_ctr; int n_zero;   // the pass's completion counters (zeroed here), or null
  // training form: per-row key ranges (RowKeys) written here
  int32_t* row_cslot; int32_t* row_blk;
  // cohort pass: the first n_draft requests run their draft rows, the others
  // their verify rows (the B drafted tokens and the last one again, so that
  // every request has B + 1 rows); drafts are kept per slot between calls
  int n_draft;
  const int32_t* phase;        // [max_batch] 0: to be drafted, 1: drafted (checked)
  const int32_t* coh_drafts;   // [max_batch, B]
  int64_t* row_off;            // [M] element offset of each row's logits
  int64_t coh_v_row0;          // logits row of the verify cohort's first row
  // tree verify pass: rows of chain j of request r form "request" r k + j
  // (B rows each); each chain keeps its keys in its scratch slot, whose page
  // table points its pages of positions c+1 .. c+B at the chain's two
  // scratch pages (written here, by the chain's first row)
  int tree_k;
  const int32_t* tree_chains;  // [n_req, k, B]
  const int32_t* tree_pages;   // [max_batch, TREE_MAX_K, 2] scratch pages
  int32_t* pt_rw;              // the page table (writable)
  int pages_per_req;
};

// a1: build the rows of a pass and gather their embeddings.
template <typename T>
__global__ void build_rows_kernel(const RowArgs a) {
  if (a.zero_ctr) {
    // after every earlier kernel has completed, before any later one starts
    pdl_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.n_zero; i += gridDim.x * blockDim.x)
      a.zero_ctr[i] = 0u;
    __threadfence();
    __syncthreads();
    pdl_trigger();
  } else {
    pdl_trigger();
    pdl_wait();
  }
  const int row = blockIdx.x;
  const int req = row / a.rows_per_req, j = row % a.rows_per_req;
  int slot, tok, pos;
  float gate = 0.f;
  if (a.kind == PASS_PREFILL) {
    slot = a.prefill_slot;
    tok = a.prompt[j];
    pos = a.prefill_pos0 + j;
  } else if (a.kind == PASS_TREE) {
    const int r = req / a.tree_k, ci = req % a.tree_k;
    int rslot = a.req_slot[r];
    if (rslot < 0 || rslot >= a.max_batch) { raise_status(a.status, ST_BAD_SLOT); rslot = 0; }
    const int c = a.cached[rslot];
    tok = a.tree_chains[((size_t)r * a.tree_k + ci) * a.B + j];
    pos = c + 1 + j;
    slot = a.max_batch + rslot * TREE_MAX_K + ci;
    if (threadIdx.x == 0) {
      a.row_cslot[row] = rslot;
      a.row_blk[row] = c + 1;
      if (j == 0) {
        const int p0 = (c + 1) / KV_PAGE;
        const int32_t* tp = a.tree_pages + ((size_t)rslot * TREE_MAX_K + ci) * 2;
        if (p0 < a.pages_per_req) a.pt_rw[(size_t)slot * a.pages_per_req + p0] = tp[0];
        if (p0 + 1 < a.pages_per_req) a.pt_rw[(size_t)slot * a.pages_per_req + p0 + 1] = tp[1];
      }
    }
  } else if (a.kind == PASS_TRAIN) {
    // training form [x, z] of sequence req: rows j < L are the clean tokens
    // x_j (gate 0, its clean slot), rows L + i the noised tokens z_i (gate on,
    // its noised slot) at the same positions; block of position i: B-aligned
    const int L = a.rows_per_req / 2;
    const bool noised = j >= L;
    const int sa = a.req_slot[2 * req], sb = a.req_slot[2 * req + 1];
    pos = noised ? j - L : j;
    tok = a.prompt[(size_t)req * a.rows_per_req + j];
    slot = noised ? sb : sa;
    gate = noised ? a.lora_scale : 0.f;
    if (threadIdx.x == 0) {
      a.row_cslot[row] = sa;
      a.row_blk[row] = noised ? (pos / a.B) * a.B : -1;
    }
  } else {
    slot = a.req_slot[req];
    if (slot < 0 || slot >= a.max_batch) { raise_status(a.status, ST_BAD_SLOT); slot = 0; }
    const int c = a.cached[slot];
    int kind = a.kind;
    if (kind == PASS_COHORT) {
      const bool draft = req < a.n_draft;
      if (a.phase[slot] != (draft ? 0 : 1)) raise_status(a.status, ST_BAD_SLOT);
      if (threadIdx.x == 0)
        a.row_off[row] = (draft ? (int64_t)slot * (a.B + 1) + j
                                : a.coh_v_row0 + (int64_t)(req - a.n_draft) * (a.B + 1) + j) * a.vocab;
      kind = draft ? PASS_DRAFT : PASS_VERIFY;
    }
    if (kind == PASS_DRAFT) {              // [pending, MASK x B] at c..c+B
      tok = (j == 0) ? a.pending[slot] : a.mask_id;
      pos = c + j;
      gate = (j == 0) ? 0.f : a.lora_scale;
    } else if (kind == PASS_VERIFY) {      // x_1..x_B at c+1..c+B
      if (a.kind == PASS_COHORT) {         // per-slot drafts; row B repeats row B-1
        const int jj = j < a.B ? j : a.B - 1;
        tok = a.coh_drafts[(size_t)slot * a.B + jj];
        pos = c + 1 + jj;
      } else {
        tok = a.drafts[(size_t)req * a.B + j];
        pos = c + 1 + j;
      }
    } else {                               // AR: pending at c
      tok = a.pending[slot];
      pos = c;
    }
  }
  if (tok < 0 || tok >= a.vocab) { raise_status(a.status, ST_BAD_TOKEN); tok = 0; }
  if (threadIdx.x == 0) {
    a.row_pos[row] = pos;
    a.row_slot[row] = slot;
    a.row_gate[row] = gate;
  }
  // embedding row -> fp32 residual, 16-byte loads, all issued up front
  constexpr int VEC = Vec16<T>::N;
  const T* e = reinterpret_cast<const T*>(a.embed) + (size_t)tok * a.d;
  float* x = a.x + (size_t)row * a.d;
  constexpr int NV = 4;
  float v[NV][VEC];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = (threadIdx.x + k * blockDim.x) * VEC;
    if (i < a.d) Vec16<T>::load(e + i, v[k]);
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = (threadIdx.x + k * blockDim.x) * VEC;
    if (i < a.d)
#pragma unroll
      for (int j = 0; j < VEC; ++j) x[i + j] = v[k][j];
  }
  for (int i = (threadIdx.x + NV * blockDim.x) * VEC; i < a.d; i += blockDim.x * VEC)
    for (int j = 0; j < VEC; ++j) x[i + j] = to_f(e[i + j]);
}

// Store y in the model dtype; with `lo` also the rounding residual
// y - round(y) (the GEMMs' split-activation rows).
template <typename T>
__device__ __forceinline__ void store_split(T* hi, T* lo, size_t i, float y) {
  const T h = from_f<T>(y);
  hi[i] = h;
  if (lo) lo[i] = from_f<T>(y - to_f(h));
}
// Four consecutive values (i a multiple of 4): one 8-byte store per row in
// bf16, one 16-byte store in fp32 (whose rounding residual is zero).
__device__ __forceinline__ void store4_split(bf16* hi, bf16* lo, size_t i, float4 y) {
  const __nv_bfloat162 h01 = __floats2bfloat162_rn(y.x, y.y), h23 = __floats2bfloat162_rn(y.z, y.w);
  uint2 hv;
  hv.x = *reinterpret_cast<const uint32_t*>(&h01);
  hv.y = *reinterpret_cast<const uint32_t*>(&h23);
  *reinterpret_cast<uint2*>(hi + i) = hv;
  if (lo) {
    const __nv_bfloat162 l01 = __floats2bfloat162_rn(y.x - __low2float(h01), y.y - __high2float(h01));
    const __nv_bfloat162 l23 = __floats2bfloat162_rn(y.z - __low2float(h23), y.w - __high2float(h23));
    uint2 lv;
    lv.x = *reinterpret_cast<const uint32_t*>(&l01);
    lv.y = *reinterpret_cast<const uint32_t*>(&l23);
    *reinterpret_cast<uint2*>(lo + i) = lv;
  }
}
__device__ __forceinline__ void store4_split(float* hi, float* lo, size_t i, float4 y) {
  *reinterpret_cast<float4*>(hi + i) = y;
  if (lo) *reinterpret_cast<float4*>(lo + i) = make_float4(0.f, 0.f, 0.f, 0.f);
}

// RMSNorm: out = x / sqrt(mean(x^2) + eps) * gain, one CTA per row.  Each
// thread holds up to RMS_V float4 of the row in registers (all loads issued
// before the reduction), so d <= 4 * NT * RMS_V.
constexpr int RMS_V = 8;
template <typename T, int NT>
__global__ void __launch_bounds__(NT) rmsnorm_kernel(const float* x, const T* gain, T* out, T* lo,
                                                     int d, int ld_out, float eps) {
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)blockIdx.x * d);
  const int n4 = d >> 2;
  float4 v[RMS_V];
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < RMS_V; ++k) {
    const int i = threadIdx.x + k * NT;
    if (i < n4) {
      v[k] = xr[i];
      s += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
    }
  }
  s = block_sum<NT>(s, red);
  const float inv = 1.0f / sqrtf(s / (float)d + eps);
  const size_t o = (size_t)blockIdx.x * ld_out;
  T* lrow = lo ? lo + o : nullptr;
#pragma unroll
  for (int k = 0; k < RMS_V; ++k) {
    const int i = threadIdx.x + k * NT;
    if (i < n4) {
      const int e = 4 * i;
      store4_split(out + o, lrow, e,
                   make_float4(v[k].x * inv * to_f(gain[e + 0]), v[k].y * inv * to_f(gain[e + 1]),
                               v[k].z * inv * to_f(gain[e + 2]), v[k].w * inv * to_f(gain[e + 3])));
    }
  }
}

// RoPE (rotate-half) on q and k of the fused fp32 qkv rows: the rotated q goes
// to q_out (the attention's input) and the rotated k and the v of every row
// into the paged pool at (slot, position), each rounded once to the
// attention operand type (KvOf).
// cos/sin come from a table [max_pos][head_dim / 2] computed on the host in
// double precision.
template <typename T>
__global__ void __launch_bounds__(256) rope_kv_kernel(const float* qkv, int ld_qkv,
                                                      typename KvOf<T>::type* q_out,
                                                      typename KvOf<T>::type* q_lo, int ld_q,
                                                      const int32_t* row_pos, const int32_t* row_slot,
                                                      const float* cos_t, const float* sin_t,
                                                      int max_pos, int H, int Hkv, int hd,
                                                      KvLayout kv, int layer, int32_t* status) {
  // one CTA per row: thread t takes the rotate-half pairs (i, i + hd/2) of
  // pair index t, t + blockDim.x, ... over the row's H + 2 Hkv heads
  // (consecutive threads, consecutive i: coalesced loads and stores).  One
  // CTA per (row, head) of hd / 2 threads had made a max-batch pass (1360
  // rows x 48 heads) bound by the launch of its 65k CTAs.
  typedef typename KvOf<T>::type KV;
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const int half = hd / 2;
  const int pos = row_pos[row], slot = row_slot[row];
  const int ok_pos = pos < max_pos;
  const int pc = ok_pos ? pos : 0;
  const float* rsrc = qkv + (size_t)row * ld_qkv;
  const int pairs = (H + 2 * Hkv) * half;
  for (int pi = threadIdx.x; pi < pairs; pi += blockDim.x) {
    const int h = pi / half, i = pi - h * half;
    const float* src = rsrc + (size_t)h * hd;
    const float x1 = src[i], x2 = src[i + half];
    if (h < H + Hkv) {
      const float c = cos_t[(size_t)pc * half + i], s = sin_t[(size_t)pc * half + i];
      const float y1 = x1 * c - x2 * s, y2 = x2 * c + x1 * s;
      if (h < H) {
        const size_t qi = (size_t)row * ld_q + (size_t)h * hd;
        const KV a1 = from_f<KV>(y1), a2 = from_f<KV>(y2);
        q_out[qi + i] = a1;
        q_out[qi + i + half] = a2;
        if (q_lo) {   // rounding residual (the attention adds q_hi K + q_lo K)
          q_lo[qi + i] = from_f<KV>(y1 - to_f(a1));
          q_lo[qi + i + half] = from_f<KV>(y2 - to_f(a2));
        }
      } else {
        int ok;
        const size_t off = kv.offset(layer, slot, pos, 0, h - H, ok);
        if (ok && ok_pos) {
          KV* dst = reinterpret_cast<KV*>(kv.pool) + off;
          const KV b1 = from_f<KV>(y1), b2 = from_f<KV>(y2);
          dst[i] = b1;
          dst[i + half] = b2;
          if (kv.n_planes == 3) {   // K lo plane
            dst[kv.plane_stride() + i] = from_f<KV>(y1 - to_f(b1));
            dst[kv.plane_stride() + i + half] = from_f<KV>(y2 - to_f(b2));
          }
        } else if (i == 0) {
          raise_status(status, ST_POS_OVERFLOW);
        }
      }
    } else {
      int ok;
      const size_t off = kv.offset(layer, slot, pos, kv.v_plane(), h - H - Hkv, ok);
      if (ok && ok_pos) {
        KV* dst = reinterpret_cast<KV*>(kv.pool) + off;
        dst[i] = from_f<KV>(x1);
        dst[i + half] = from_f<KV>(x2);
      }
    }
  }
}

// SwiGLU: out[:, f] = silu(gu[:, f]) * gu[:, F + f], from the fp32 gate|up rows.
// Grid (rows, ceil(F / (4 * blockDim))): each thread does 4 consecutive
// features with one float4 load of gate and one of up.
template <typename T>
__global__ void swiglu_kernel(const float* gu, int F, T* out, T* lo) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const int f = 4 * (blockIdx.y * blockDim.x + threadIdx.x);
  if (f >= F) return;
  const float* g = gu + (size_t)row * 2 * F;
  const float4 a = *reinterpret_cast<const float4*>(g + f);
  const float4 b = *reinterpret_cast<const float4*>(g + F + f);
  const size_t o = (size_t)row * F + f;
  T* lrow = lo ? lo + o : nullptr;
  store4_split(out + o, lrow, 0,
               make_float4(a.x / (1.0f + expf(-a.x)) * b.x, a.y / (1.0f + expf(-a.y)) * b.y,
                           a.z / (1.0f + expf(-a.z)) * b.z, a.w / (1.0f + expf(-a.w)) * b.w));
}

// Prefill bookkeeping: cached = P - 1, pending = prompt[P - 1].
__global__ void init_slot_kernel(const int32_t* prompt, int P, int slot, int32_t* cached,
                                 int32_t* pending) {
  pdl_trigger();
  pdl_wait();
  cached[slot] = P - 1;
  pending[slot] = prompt[P - 1];
}

}  // namespace uno
