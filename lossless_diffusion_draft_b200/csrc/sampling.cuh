// Sampling kernels of the Psi-Spec iteration: draft_sample (first token from
// the AR row, drafts 2..B from the diffusion rows), the AR-only sampler, and
// spec_verify (accept tests, first-rejection prefix, residual redraw or bonus
// token, commit).
//
// Method (blog page "不砸掉重来，给自回归 LLM 装一对“扩散翅膀”：Uno 的无损加速之路",
// section Ψ-Spec 采样器：起草、验证、两种模式): the block's first token comes from
// the AR weights alone and is always kept; the AR path verifies the whole
// block, the longest accepted prefix is kept and the first rejected position
// is redrawn from the renormalised residual max(0, p - q).
//
// Work split.  A vocabulary row is cut into chunks of `ch` logits; one CTA
// reduces one (row, chunk) to its (max, sum exp(l - max)) pair.  The last CTA
// to finish a row (atomic counter, no waiting) combines the row's pairs in
// chunk order; the last row of a request runs the request's decision.  A
// rejected request's residual is summed by a second grid, one CTA per
// (request, chunk), whose last CTA draws the token.  No CTA ever waits on
// another, so nothing can hang.
//
// Inverse-CDF sampling on the device: w_v = exp(l_v - M) with M the row max
// (exp_rel below); Z = sum over chunks (a chunk-order scan) of
// s_k * expf(m_k - M), s_k the chunk's sum relative to its own max m_k; the token is in
// the first chunk whose running prefix exceeds u * Z, at the first element
// whose within-chunk inclusive prefix (thread-contiguous order, fixed) pushes
// the running sum above u * Z.  When rounding leaves no crossing, the last
// element with positive weight (of the chunk, or of the row) is taken.
#pragma once

#include <climits>

#include "common.cuh"

namespace uno {

constexpr int SAMPLE_THREADS = 256;

// exp(x - m) as 2^(x log2 e - m log2 e): one FMA (mL = m log2 e, computed
// once per row or chunk) and the special-function unit's ex2.approx (about
// 2 ulp).  The rounding of mL scales every weight of the row or chunk by the
// same factor (relative 1e-6 at |m| ~ 20), which the normaliser divides out.
// Every per-logit exponential of this file goes through here, so the chunk
// sums and the element weights of the crossing scan use the same values.
constexpr float SAMPLE_LOG2E = 1.4426950408889634f;
__device__ __forceinline__ float exp_rel(float x, float mL) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(fmaf(x, SAMPLE_LOG2E, -mL)));
  return y;
}

// ---------------------------------------------------------------------------
// Nucleus (top-p) filter of a row (blog page "…Uno 的无损加速之路", section
// 我的判断: the lossless claim holds for the sampling distribution of
// temperature 1 and top-p 0.95).  The nucleus is the smallest set of the most
// probable tokens whose probability reaches top_p, tokens ordered by
// probability with ties by token id; it is stored per row as an
// order-preserving 32-bit key of the crossing logit and the last token id
// kept among the tokens with exactly that logit.  Every kernel below reads a
// filtered logit as l if the token is kept and -inf otherwise, so the
// softmax of the filtered row is the renormalised nucleus distribution.
// ---------------------------------------------------------------------------
struct RowFilter { uint32_t key; int32_t id_cut; };
// key(l) orders floats like their values: higher logit, higher key
__device__ __forceinline__ uint32_t logit_key(float l) {
  uint32_t u = __float_as_uint(l);
  if (u == 0x80000000u) u = 0u;   // -0 and +0 are one value
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
// FILT = false: no filter (compiled out).
template <bool FILT>
struct Filt {
  uint32_t key; int32_t id_cut;
  __device__ __forceinline__ float operator()(float l, int v) const {
    if (!FILT) return l;
    const uint32_t k = logit_key(l);
    return (k > key || (k == key && v <= id_cut)) ? l : -INFINITY;
  }
  __device__ __forceinline__ float4 four(float4 x, int v) const {
    if (!FILT) return x;
    return make_float4((*this)(x.x, v), (*this)(x.y, v + 1), (*this)(x.z, v + 2), (*this)(x.w, v + 3));
  }
};
template <bool FILT>
__device__ __forceinline__ Filt<FILT> filt_of(const RowFilter* f, size_t row) {
  if (!FILT || !f) return Filt<FILT>{0u, -1};
  const RowFilter r = f[row];
  return Filt<FILT>{r.key, r.id_cut};
}

// ---------------------------------------------------------------------------
// Phase A: reduce one chunk of one row to (max, sum exp(l - max)).  The
// CTA's max comes first (warp butterfly, then the warps' maxima in order),
// then every logit takes one exponential against it and the sums are added
// by a butterfly and the warps in order: a fixed tree, and no rescaling.
// ---------------------------------------------------------------------------
constexpr int CHUNK_IT = 8;   // float4 per thread: a chunk holds <= 8 * 4 * 256 = 8192 logits
// A thread's loads of a chunk (16 bytes each, streaming; rows start on
// 16-byte boundaries: vocab % 4 == 0 is required), the filter applied.
template <bool FILT>
__device__ __forceinline__ void chunk_load(const float* row, int c0, int c1, float4 (&v)[CHUNK_IT],
                                           Filt<FILT> f) {
  const int n4 = (c1 - c0) >> 2;
  const float4* r4 = reinterpret_cast<const float4*>(row + c0);
#pragma unroll
  for (int i = 0; i < CHUNK_IT; ++i) {
    const int j = threadIdx.x + i * SAMPLE_THREADS;
    if (j < n4) v[i] = f.four(__ldcs(r4 + j), c0 + 4 * j);
  }
}
// The reduction of a chunk whose float4 part chunk_load has brought into v.
// red: at least 2 * SAMPLE_THREADS / 32 floats of shared memory.
template <bool FILT>
__device__ __forceinline__ float2 chunk_reduce(const float* row, int c0, int c1,
                                               const float4 (&v)[CHUNK_IT], float* red, Filt<FILT> f) {
  constexpr int NW = SAMPLE_THREADS / 32;
  const int n4 = (c1 - c0) >> 2;
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < CHUNK_IT; ++i) {
    const int j = threadIdx.x + i * SAMPLE_THREADS;
    if (j < n4) m = fmaxf(m, fmaxf(fmaxf(v[i].x, v[i].y), fmaxf(v[i].z, v[i].w)));
  }
  // scalar tail (chunk length not a multiple of 4: only the row's last chunk)
  for (int j = c0 + (n4 << 2) + threadIdx.x; j < c1; j += SAMPLE_THREADS) m = fmaxf(m, f(row[j], j));
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();                                    // red may hold a previous reduction
  if (lane == 0) red[wid] = m;
  __syncthreads();
  float M = red[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, red[w]);
  float s = 0.f;
  if (M != -INFINITY) {
    const float mL = M * SAMPLE_LOG2E;
#pragma unroll
    for (int i = 0; i < CHUNK_IT; ++i) {
      const int j = threadIdx.x + i * SAMPLE_THREADS;
      if (j < n4)
        s += (exp_rel(v[i].x, mL) + exp_rel(v[i].y, mL)) + (exp_rel(v[i].z, mL) + exp_rel(v[i].w, mL));
    }
    for (int j = c0 + (n4 << 2) + threadIdx.x; j < c1; j += SAMPLE_THREADS) s += exp_rel(f(row[j], j), mL);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[NW + wid] = s;                   // other slots than the maxima
  __syncthreads();
  float S = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) S += red[NW + w];
  return make_float2(M, S);
}
template <bool FILT = false>
__device__ __forceinline__ float2 reduce_chunk(const float* row, int c0, int c1, float* red,
                                               Filt<FILT> f = Filt<FILT>{0u, -1}) {
  float4 v[CHUNK_IT];
  chunk_load<FILT>(row, c0, c1, v, f);
  return chunk_reduce<FILT>(row, c0, c1, v, red, f);
}

// Chunk-level prefix in chunk order, run by one whole warp: lane l holds
// chunks l, l + 32, ...; each group of 32 is scanned with shuffles (fixed
// tree) and carried into the next.  Returns on every lane: the first chunk
// whose inclusive prefix exceeds `target` (-1 if none) with its exclusive
// prefix, the last chunk of positive weight (-1 if none) and the total.
// Every caller that needs the row's Z and its running prefix goes through
// this one routine, so the two agree bit for bit.
struct ChunkPick { int k; float base; int lastk; float total; };
template <typename F>
__device__ __forceinline__ ChunkPick warp_chunk_pick(const F& wk, int nch, float target) {
  const int lane = threadIdx.x & 31;
  ChunkPick r{-1, 0.f, -1, 0.f};
  float carry = 0.f;
  for (int g = 0; g < nch; g += 32) {
    const int c = g + lane;
    const float w = c < nch ? wk(c) : 0.f;
    float incl = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.f;
    incl += carry;
    excl += carry;
    const unsigned hit = __ballot_sync(0xffffffffu, c < nch && incl > target);
    if (r.k < 0 && hit) {
      const int l = __ffs(hit) - 1;
      r.k = g + l;
      r.base = __shfl_sync(0xffffffffu, excl, l);
    }
    const unsigned pos = __ballot_sync(0xffffffffu, c < nch && w > 0.f);
    if (pos) r.lastk = g + 31 - __clz(pos);
    carry = __shfl_sync(0xffffffffu, incl, 31);
  }
  r.total = carry;
  return r;
}

// Weight of chunk k relative to the row max M: s_k * exp(m_k - M).
struct ChunkW {
  const float2* part; float M;
  __device__ __forceinline__ float operator()(int k) const {
    const float2 pk = __ldcg(&part[k]);
    return pk.x != -INFINITY ? pk.y * expf(pk.x - M) : 0.f;
  }
};

// Row-level combine of chunk pairs (one whole warp; the result on every lane).
struct RowStat { float M, Z; };
// Plain per-chunk sums (the residual's).
struct PartW {
  const float* s;
  __device__ __forceinline__ float operator()(int k) const { return __ldcg(&s[k]); }
};
__device__ __forceinline__ RowStat combine_row(const float2* part, int nch) {
  const int lane = threadIdx.x & 31;
  float M = -INFINITY;
  for (int k = lane; k < nch; k += 32) M = fmaxf(M, __ldcg(&part[k].x));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (M == -INFINITY) return {M, 0.f};
  const ChunkPick cp = warp_chunk_pick(ChunkW{part, M}, nch, INFINITY);
  return {M, cp.total};
}

// Weight functors used by the crossing scan (get4: four weights from v, a
// multiple of 4).
template <bool FILT = false>
struct SoftmaxW {
  const float* row; float ML;          // row max x log2 e
  Filt<FILT> f;
  __device__ __forceinline__ float operator()(int v) const { return exp_rel(f(row[v], v), ML); }
  __device__ __forceinline__ void get4(int v, float* w) const {
    const float4 x = f.four(*reinterpret_cast<const float4*>(row + v), v);
    w[0] = exp_rel(x.x, ML); w[1] = exp_rel(x.y, ML); w[2] = exp_rel(x.z, ML); w[3] = exp_rel(x.w, ML);
  }
};
template <bool FILT = false>
struct ResidW {
  const float* p; const float* q; float lpL, lqL;   // lse_p, lse_q x log2 e
  Filt<FILT> fp, fq;
  __device__ __forceinline__ float pair(float pv, float qv, int v) const {
    const float d = exp_rel(fp(pv, v), lpL) - exp_rel(fq(qv, v), lqL);
    return d > 0.f ? d : 0.f;
  }
  __device__ __forceinline__ float operator()(int v) const { return pair(p[v], q[v], v); }
  __device__ __forceinline__ void get4(int v, float* w) const {
    const float4 x = *reinterpret_cast<const float4*>(p + v);
    const float4 y = *reinterpret_cast<const float4*>(q + v);
    w[0] = pair(x.x, y.x, v); w[1] = pair(x.y, y.y, v + 1); w[2] = pair(x.z, y.z, v + 2);
    w[3] = pair(x.w, y.w, v + 3);
  }
};

// First v in [c0, c1) whose running prefix base + sum_{c0..v} w exceeds
// target (thread-contiguous segments of a multiple of 4 elements, fixed
// order); -1 if none.  `last_pos` receives the last v with w > 0 (-1 if
// none).  c0 and c1 are multiples of 4 and c1 - c0 <= 4 * CHUNK_IT *
// SAMPLE_THREADS.  Each thread reads its segment once (16-byte loads) and
// keeps the weights in registers for the scan.  All threads participate.
template <typename W>
__device__ int chunk_crossing(const W& w, int c0, int c1, float base, float target, int* last_pos,
                              float* red) {
  constexpr int SEG = 4 * CHUNK_IT;   // elements per thread at most
  __shared__ float s_tot[SAMPLE_THREADS / 32];
  __shared__ int s_i[2];
  const int len = c1 - c0;
  const int per = ((len + 4 * SAMPLE_THREADS - 1) / (4 * SAMPLE_THREADS)) * 4;
  const int b = c0 + threadIdx.x * per;
  const int e = min(c1, b + per);
  float wv[SEG];
#pragma unroll
  for (int k = 0; k < SEG; k += 4) {
    if (b + k < e) w.get4(b + k, wv + k);
    else wv[k] = wv[k + 1] = wv[k + 2] = wv[k + 3] = 0.f;
  }
  float tsum = 0.f;
  int lastpos = -1;
#pragma unroll
  for (int k = 0; k < SEG; ++k) {
    tsum += wv[k];
    if (wv[k] > 0.f) lastpos = b + k;
  }
  // block exclusive scan of tsum
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float incl = tsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (threadIdx.x == 0) { s_i[0] = INT_MAX; s_i[1] = -1; }
  if (lane == 31) s_tot[wid] = incl;
  __syncthreads();
  float wbase = 0.f;
  for (int k = 0; k < wid; ++k) wbase += s_tot[k];
  float run = base + wbase + (incl - tsum);
  int hit = INT_MAX;
#pragma unroll
  for (int k = 0; k < SEG; ++k) {
    run += wv[k];
    if (hit == INT_MAX && b + k < e && run > target) hit = b + k;
  }
  if (hit != INT_MAX) atomicMin(&s_i[0], hit);
  if (lastpos >= 0) atomicMax(&s_i[1], lastpos);
  __syncthreads();
  const int r = s_i[0];
  *last_pos = s_i[1];
  __syncthreads();
  (void)red;
  return r == INT_MAX ? -1 : r;
}

// Sample a softmax row from its chunk pairs with uniform u (whole CTA).
template <bool FILT = false>
__device__ int sample_from_partials(const float* row, const float2* part, int nch, int ch, int V,
                                    const RowStat& rs, float u, float* red,
                                    Filt<FILT> f = Filt<FILT>{0u, -1}) {
  __shared__ int s_k;
  __shared__ float s_base;
  const float target = u * rs.Z;
  if (threadIdx.x < 32) {
    ChunkPick cp{-1, 0.f, -1, 0.f};
    if (rs.M != -INFINITY) cp = warp_chunk_pick(ChunkW{part, rs.M}, nch, target);
    if (cp.k < 0) { cp.k = cp.lastk; cp.base = 0.f; }
    if (threadIdx.x == 0) { s_k = cp.k; s_base = cp.base; }
  }
  __syncthreads();
  const int k = s_k;
  const float base = s_base;
  __syncthreads();
  if (k < 0) return 0;  // empty row (all -inf): only reachable with invalid logits
  SoftmaxW<FILT> w{row, rs.M * SAMPLE_LOG2E, f};
  int lastpos;
  const int c0 = k * ch, c1 = min(V, c0 + ch);
  int t = chunk_crossing(w, c0, c1, base, target, &lastpos, red);
  if (t < 0) t = lastpos >= 0 ? lastpos : c0;
  return t;
}

// ---------------------------------------------------------------------------
// draft_sample / AR sample.
// ---------------------------------------------------------------------------
struct SampleArgs {
  const float* logits;        // [n_req, logit_rows_per_req, V]
  int V, nch, ch;
  int rows_per_req;           // sampled rows per request
  int logit_rows_per_req;
  int ar_mode;                // 0: draft (row 0 FIRST, sampled row s>0 reads logits row s+1, DRAFT)
                              // 1: AR step (row 0 FIRST, commits the token)
  const int32_t* req_slot;    // [n_req] slot ids
  int32_t* cached;            // [max_batch] cached token count per slot
  int32_t* pending;           // [max_batch] pending token per slot
  const uint32_t* slot_stream;
  uint64_t seed;
  int32_t* out_tok; int out_stride;   // draft: [n_req, rows_per_req]; AR: [n_req]
  float* lse_out;             // [n_req, rows_per_req] or null
  float2* partial;            // [n_req * rows_per_req, nch]
  unsigned* row_counter;      // [n_req * rows_per_req], zero on entry, left zero
  int32_t* status;
  const RowFilter* filt;      // nucleus of each logit row [n_req * logit_rows_per_req] (FILT)
  // per_slot: logits, drafts, lse and filters are indexed by the request's
  // slot instead of its position in the batch (the cohort step keeps them
  // between calls), and phase[slot] is set to 1 (drafted)
  int per_slot; int32_t* phase;
  // tree sampler (tree_k >= 1): sampled row 0 is x_1, row 1 + j (B-1) + d - 2
  // draws chain j's token at position c + d from logit row d with Philox lane
  // j; out_tok is [n_req, tree_k, B] (x_1 at index 0 of every chain), and
  // lse_out [n_req, B] keeps lse(q_d) at index d - 1 (from chain 0's rows)
  int tree_k, tree_B;
};

template <bool FILT>
__global__ void __launch_bounds__(SAMPLE_THREADS, 3) sample_rows_kernel(const SampleArgs a) {
  __shared__ float red[32];
  __shared__ bool s_last;
  pdl_trigger();
  pdl_wait();
  const int k = blockIdx.x;
  const int rid = blockIdx.y;
  const int req = rid / a.rows_per_req, s = rid % a.rows_per_req;
  int lrow = (a.ar_mode || s == 0) ? 0 : s + 1;
  int lane = 0;
  if (a.tree_k > 0 && s > 0) {
    lane = (s - 1) / (a.tree_B - 1);
    lrow = 2 + (s - 1) % (a.tree_B - 1);
  }
  const int slot = a.req_slot[req];
  const int base = a.per_slot ? slot : req;
  const float* row = a.logits + ((size_t)base * a.logit_rows_per_req + lrow) * a.V;
  const Filt<FILT> f = filt_of<FILT>(a.filt, (size_t)base * a.logit_rows_per_req + lrow);
  const int c0 = k * a.ch, c1 = min(a.V, c0 + a.ch);
  const float2 pr = reduce_chunk<FILT>(row, c0, c1, red, f);
  if (threadIdx.x == 0) {
    a.partial[(size_t)rid * a.nch + k] = pr;
    __threadfence();
    const unsigned done = atomicAdd(&a.row_counter[rid], 1u);
    s_last = (done == (unsigned)a.nch - 1);
    if (s_last) a.row_counter[rid] = 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float2* part = a.partial + (size_t)rid * a.nch;
  __shared__ RowStat s_rs;
  if (threadIdx.x < 32) {
    const RowStat rs = combine_row(part, a.nch);
    if (threadIdx.x == 0) s_rs = rs;
  }
  __syncthreads();
  const RowStat rs = s_rs;
  const int c = a.cached[slot];
  const uint32_t kind = (a.ar_mode || s == 0) ? KIND_FIRST : KIND_DRAFT;
  // the token at position c + 1 (x_1) or c + d (logit row d)
  const int pos = (a.ar_mode || s == 0) ? c + 1 : c + lrow;
  const float u = philox_uniform(a.seed, a.slot_stream[slot], (uint32_t)pos, kind, (uint32_t)lane);
  const int t = sample_from_partials<FILT>(row, part, a.nch, a.ch, a.V, rs, u, red, f);
  if (threadIdx.x == 0) {
    if (a.ar_mode) {
      a.out_tok[req] = t;
      a.cached[slot] = c + 1;
      a.pending[slot] = t;
    } else if (a.tree_k > 0) {
      const int B = a.tree_B;
      if (s == 0) {
        for (int j = 0; j < a.tree_k; ++j) a.out_tok[((size_t)req * a.tree_k + j) * B] = t;
      } else {
        a.out_tok[((size_t)req * a.tree_k + lane) * B + lrow - 1] = t;
        if (lane == 0 && a.lse_out) a.lse_out[(size_t)req * B + lrow - 1] = rs.M + logf(rs.Z);
      }
    } else {
      a.out_tok[(size_t)base * a.out_stride + s] = t;
      if (a.lse_out) a.lse_out[(size_t)base * a.rows_per_req + s] = rs.M + logf(rs.Z);
      if (a.phase && s == 0) a.phase[slot] = 1;
    }
  }
}

// ---------------------------------------------------------------------------
// spec_verify.
// ---------------------------------------------------------------------------
struct VerifyArgs {
  const float* p; const float* q;
  int V, nch, ch;
  int n_tests;                 // drafted tokens tested per request
  int64_t p_req_rows, q_req_rows;   // rows per request in p / q buffers
  int p_row0, q_row0;          // buffer row of test 0
  int bonus_row;               // p buffer row of the bonus distribution, -1: none
  const int32_t* drafts; int drafts_stride, drafts_off;   // token of test j
  const float* lse_q_in; int lse_q_stride, lse_q_off;     // optional lse of q rows
  uint64_t seed;
  // decode mode (req_slot != null): state lives per slot
  const int32_t* req_slot; int32_t* cached; int32_t* pending; const uint32_t* slot_stream;
  int32_t* first_tok;          // decode mode: x_1 per request (drafts[i*stride + 0])
  // stand-alone mode
  const uint32_t* streams; const int32_t* pos0;
  int32_t* out_tok; int out_stride; int32_t* n_out;
  // workspace
  float2* partial;             // [n_req * rows_red, nch]
  float* lse;                  // [n_req * rows_red]
  unsigned* row_counter;       // [n_req * rows_red]
  unsigned* req_counter;       // [n_req]
  int32_t* at_ws;              // [n_req] first rejected test, -1: finished by the first stage
  float* resid_part;           // [n_req, nch] residual chunk sums
  unsigned* resid_counter;     // [n_req]
  int rows_red;                // rows reduced per request
  int n_p;                     // of which p rows (tests + bonus)
  int32_t* status;
  // benchmark tap (-1: off): the accepted prefix is forced to min(fixed_at,
  // n_tests) tests instead of the accept tests' outcome; the residual
  // redraw or the bonus draw then runs as usual
  int fixed_at;
  // nucleus of each p row [n_req * p_req_rows] and q row [n_req * q_req_rows] (FILT)
  const RowFilter* filt_p; const RowFilter* filt_q;
  // per_slot (decode mode): q rows, drafts, their lse and filters are indexed
  // by the request's slot (kept there by the cohort step's draft_sample), and
  // phase[slot] is reset to 0 at the commit
  int per_slot; int32_t* phase;
};
// Index of a request's draft-side data (q rows, drafts, lse of q).
__device__ __forceinline__ int verify_qb(const VerifyArgs& a, int req) {
  return a.per_slot ? a.req_slot[req] : req;
}

// Slot, position of test 0 and Philox stream of a request.
__device__ __forceinline__ void verify_request_ctx(const VerifyArgs& a, int req, int* slot,
                                                   int* pos0, uint32_t* stream) {
  if (a.req_slot) {
    *slot = a.req_slot[req];
    *pos0 = a.cached[*slot] + 2;     // test 0 is x_2 at position c + 2
    *stream = a.slot_stream[*slot];
  } else {
    *slot = -1;
    *pos0 = a.pos0[req];
    *stream = a.streams[req];
  }
}

// log-normaliser of the draft row of test j.
__device__ __forceinline__ float verify_lse_q(const VerifyArgs& a, int req, int j) {
  return a.lse_q_in ? a.lse_q_in[(size_t)verify_qb(a, req) * a.lse_q_stride + a.lse_q_off + j]
                    : __ldcg(&a.lse[(size_t)req * a.rows_red + a.n_p + j]);
}

// Outputs and commit of a request with `at` accepted tests and final token y
// (whole CTA).
__device__ void verify_finish(const VerifyArgs& a, int req, int slot, int pos0, int at, int y) {
  const bool decode = a.req_slot != nullptr;
  const int lead = decode ? 1 : 0;    // decode mode emits x_1 first
  int32_t* out = a.out_tok + (size_t)req * a.out_stride;
  const int qb = verify_qb(a, req);
  for (int j = threadIdx.x; j < at; j += SAMPLE_THREADS)
    out[lead + j] = a.drafts[(size_t)qb * a.drafts_stride + a.drafts_off + j];
  if (threadIdx.x == 0) {
    if (decode) {
      // emitted: x_1, the accepted x_2..x_{1+at}, then y; the cache grows by
      // n tokens (positions c..c+n-1 hold keys/values) and y becomes pending
      out[0] = a.first_tok[(size_t)qb * a.drafts_stride];
      const int n = lead + at + 1;
      out[n - 1] = y;
      a.n_out[req] = n;
      a.cached[slot] = pos0 - 2 + n;
      a.pending[slot] = y;
      if (a.phase) a.phase[slot] = 0;
    } else {
      out[at] = y;          // -1 when every test passed and no bonus row exists
      a.n_out[req] = at;
    }
  }
}

// The decision of request req once every reduced row's lse is in a.lse
// (whole CTA): the accept tests, the first rejection, and either the bonus
// draw and the commit here or the hand-over to spec_resid_kernel.
template <bool FILT>
__device__ __forceinline__ Filt<FILT> verify_filt_p(const VerifyArgs& a, int req, int prow_idx) {
  return filt_of<FILT>(a.filt_p, (size_t)req * a.p_req_rows + prow_idx);
}
template <bool FILT>
__device__ __forceinline__ Filt<FILT> verify_filt_q(const VerifyArgs& a, int req, int qrow_idx) {
  return filt_of<FILT>(a.filt_q, (size_t)verify_qb(a, req) * a.q_req_rows + qrow_idx);
}

template <bool FILT>
__device__ void verify_decide(const VerifyArgs& a, int req, float* red) {
  __shared__ int s_a;
  const size_t rbase = (size_t)req * a.rows_red;
  int slot, pos0;
  uint32_t stream;
  verify_request_ctx(a, req, &slot, &pos0, &stream);
  if (threadIdx.x == 0) s_a = a.n_tests;
  __syncthreads();
  const int qb = verify_qb(a, req);
  for (int j = threadIdx.x; j < a.n_tests; j += SAMPLE_THREADS) {
    int t = a.drafts[(size_t)qb * a.drafts_stride + a.drafts_off + j];
    if (t < 0 || t >= a.V) { raise_status(a.status, ST_BAD_TOKEN); t = 0; }
    const float* prow = a.p + ((size_t)req * a.p_req_rows + a.p_row0 + j) * a.V;
    const float* qrow = a.q + ((size_t)qb * a.q_req_rows + a.q_row0 + j) * a.V;
    const float lse_p = __ldcg(&a.lse[rbase + j]);
    const float lse_q = verify_lse_q(a, req, j);
    const float u = philox_uniform(a.seed, stream, (uint32_t)(pos0 + j), KIND_ACCEPT);
    const float lp = verify_filt_p<FILT>(a, req, a.p_row0 + j)(prow[t], t);
    const float lq = verify_filt_q<FILT>(a, req, a.q_row0 + j)(qrow[t], t);
    const bool acc = logf(u) < (lp - lse_p) - (lq - lse_q);
    if (!acc) atomicMin(&s_a, j);
  }
  __syncthreads();
  const int at = a.fixed_at >= 0 ? min(a.fixed_at, a.n_tests) : s_a;   // accepted tests
  if (at < a.n_tests) {
    // a rejection: spec_resid_kernel draws from the residual and finishes
    if (threadIdx.x == 0) a.at_ws[req] = at;
    return;
  }
  int y = -1;
  if (a.bonus_row >= 0) {
    const float* prow = a.p + ((size_t)req * a.p_req_rows + a.bonus_row) * a.V;
    const float u = philox_uniform(a.seed, stream, (uint32_t)(pos0 + a.n_tests), KIND_RESID);
    __shared__ RowStat s_rs2;
    if (threadIdx.x < 32) {
      const RowStat rs = combine_row(a.partial + (rbase + a.n_tests) * a.nch, a.nch);
      if (threadIdx.x == 0) s_rs2 = rs;
    }
    __syncthreads();
    y = sample_from_partials<FILT>(prow, a.partial + (rbase + a.n_tests) * a.nch, a.nch, a.ch, a.V,
                                   s_rs2, u, red, verify_filt_p<FILT>(a, req, a.bonus_row));
  }
  if (threadIdx.x == 0) a.at_ws[req] = -1;
  verify_finish(a, req, slot, pos0, at, y);
}

// The row a (request, reduced row) CTA reads.
__device__ __forceinline__ const float* verify_row(const VerifyArgs& a, int req, int r) {
  if (r < a.n_p) {
    const int br = (r < a.n_tests) ? a.p_row0 + r : a.bonus_row;
    return a.p + ((size_t)req * a.p_req_rows + br) * a.V;
  }
  return a.q + ((size_t)verify_qb(a, req) * a.q_req_rows + a.q_row0 + (r - a.n_p)) * a.V;
}

// The nucleus of the row a (request, reduced row) CTA reads.
template <bool FILT>
__device__ __forceinline__ Filt<FILT> verify_row_filt(const VerifyArgs& a, int req, int r) {
  if (r < a.n_p) return verify_filt_p<FILT>(a, req, (r < a.n_tests) ? a.p_row0 + r : a.bonus_row);
  return verify_filt_q<FILT>(a, req, a.q_row0 + (r - a.n_p));
}

// Fused form (few rows): grid (nch, n_req * rows_red).  The last chunk CTA
// of a row forms its lse, the last row of a request decides.
template <bool FILT>
__global__ void __launch_bounds__(SAMPLE_THREADS, 3) spec_verify_kernel(const VerifyArgs a) {
  __shared__ float red[32];
  __shared__ bool s_last, s_req_last;
  pdl_trigger();
  pdl_wait();
  const int k = blockIdx.x;
  const int rid = blockIdx.y;
  const int req = rid / a.rows_red, r = rid % a.rows_red;
  const float* row = verify_row(a, req, r);
  const int c0 = k * a.ch, c1 = min(a.V, c0 + a.ch);
  const float2 pr = reduce_chunk<FILT>(row, c0, c1, red, verify_row_filt<FILT>(a, req, r));
  if (threadIdx.x == 0) {
    a.partial[(size_t)rid * a.nch + k] = pr;
    __threadfence();
    const unsigned done = atomicAdd(&a.row_counter[rid], 1u);
    s_last = (done == (unsigned)a.nch - 1);
    if (s_last) a.row_counter[rid] = 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last chunk of the row: its lse; the last row of the request decides
  if (threadIdx.x < 32) {
    const RowStat rs = combine_row(a.partial + (size_t)rid * a.nch, a.nch);
    if (threadIdx.x == 0) {
      a.lse[rid] = rs.M + logf(rs.Z);
      __threadfence();
      const unsigned rdone = atomicAdd(&a.req_counter[req], 1u);
      s_req_last = (rdone == (unsigned)a.rows_red - 1);
      if (s_req_last) a.req_counter[req] = 0u;
    }
  }
  __syncthreads();
  if (!s_req_last) return;
  __threadfence();
  verify_decide<FILT>(a, req, red);
}

// Split form (many rows), first kernel: grid (ceil(nch / 2), n_req *
// rows_red), every CTA reduces two consecutive chunks of a row, writes their
// pairs and exits (no counters, no waiting on a round trip).  Both chunks'
// loads are issued before either is reduced, so an SM keeps its three CTAs'
// 64 KB each in flight through the reductions (measured on 4096 x 151936
// fp32 p and q: 0.752 ms against 0.957 with one chunk a CTA at four CTAs an
// SM, and 1.29 / 1.18 ms at five / six).
template <bool FILT>
__global__ void __launch_bounds__(SAMPLE_THREADS, 3) spec_reduce_kernel(const VerifyArgs a) {
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const int k0 = 2 * blockIdx.x;
  const int rid = blockIdx.y;
  const int req = rid / a.rows_red, r = rid % a.rows_red;
  const float* row = verify_row(a, req, r);
  const Filt<FILT> f = verify_row_filt<FILT>(a, req, r);
  const int c0 = k0 * a.ch, c1 = min(a.V, c0 + a.ch);
  const bool two = k0 + 1 < a.nch;
  const int d1 = min(a.V, c1 + a.ch);
  float4 v0[CHUNK_IT], v1[CHUNK_IT];
  chunk_load<FILT>(row, c0, c1, v0, f);
  if (two) chunk_load<FILT>(row, c1, d1, v1, f);
  const float2 p0 = chunk_reduce<FILT>(row, c0, c1, v0, red, f);
  if (threadIdx.x == 0) a.partial[(size_t)rid * a.nch + k0] = p0;
  if (two) {
    const float2 p1 = chunk_reduce<FILT>(row, c1, d1, v1, red, f);
    if (threadIdx.x == 0) a.partial[(size_t)rid * a.nch + k0 + 1] = p1;
  }
}

// Split form, second kernel: one CTA per request; warp w forms the lse of
// rows w, w + 8, ... (the same chunk-order combine as the fused form), then
// the CTA decides.
template <bool FILT>
__global__ void __launch_bounds__(SAMPLE_THREADS) spec_decide_kernel(const VerifyArgs a) {
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const int req = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  for (int r = warp; r < a.rows_red; r += SAMPLE_THREADS / 32) {
    const size_t rid = (size_t)req * a.rows_red + r;
    const RowStat rs = combine_row(a.partial + rid * a.nch, a.nch);
    if ((threadIdx.x & 31) == 0) a.lse[rid] = rs.M + logf(rs.Z);
  }
  __syncthreads();
  verify_decide<FILT>(a, req, red);
}

// ---------------------------------------------------------------------------
// spec_verify, second stage: the residual redraw at the first rejected test.
// Grid (nch, n_req); launched after spec_verify_kernel.  CTA k adds up the
// residual weights max(0, p_v - q_v) (normalised p and q of the rejected
// test's rows) over chunk k; the last CTA of a request picks the chunk whose
// running sum (chunk order) crosses u * Z, finds the token inside it, and
// writes the outputs and the commit.  Requests without a rejection (at_ws =
// -1) were finished by the first stage.
// ---------------------------------------------------------------------------
template <bool FILT>
__global__ void __launch_bounds__(SAMPLE_THREADS) spec_resid_kernel(const VerifyArgs a) {
  __shared__ float red[32];
  __shared__ bool s_last;
  pdl_trigger();
  pdl_wait();
  const int k = blockIdx.x, req = blockIdx.y;
  const int at = a.at_ws[req];
  if (at < 0) return;
  const size_t rbase = (size_t)req * a.rows_red;
  const float* prow = a.p + ((size_t)req * a.p_req_rows + a.p_row0 + at) * a.V;
  const float* qrow = a.q + ((size_t)verify_qb(a, req) * a.q_req_rows + a.q_row0 + at) * a.V;
  const float lse_p = __ldcg(&a.lse[rbase + at]);
  const float lse_q = verify_lse_q(a, req, at);
  const Filt<FILT> fp = verify_filt_p<FILT>(a, req, a.p_row0 + at);
  const ResidW<FILT> w{prow, qrow, lse_p * SAMPLE_LOG2E, lse_q * SAMPLE_LOG2E, fp,
                       verify_filt_q<FILT>(a, req, a.q_row0 + at)};
  {
    // chunk sum: 16-byte loads, all of a thread's loads issued first
    const int b0 = k * a.ch, b1 = min(a.V, b0 + a.ch);
    const int n4 = (b1 - b0) >> 2;
    const float4* p4 = reinterpret_cast<const float4*>(prow + b0);
    const float4* q4 = reinterpret_cast<const float4*>(qrow + b0);
    constexpr int MAXIT = 8;
    float sacc = 0.f;
    for (int i0 = 0; i0 < n4; i0 += MAXIT * SAMPLE_THREADS) {
      float4 x[MAXIT], z[MAXIT];
#pragma unroll
      for (int i = 0; i < MAXIT; ++i) {
        const int j = i0 + threadIdx.x + i * SAMPLE_THREADS;
        if (j < n4) { x[i] = p4[j]; z[i] = q4[j]; }
      }
#pragma unroll
      for (int i = 0; i < MAXIT; ++i) {
        const int j = i0 + threadIdx.x + i * SAMPLE_THREADS;
        const int v = b0 + 4 * j;
        if (j < n4) sacc += w.pair(x[i].x, z[i].x, v) + w.pair(x[i].y, z[i].y, v + 1) +
                            w.pair(x[i].z, z[i].z, v + 2) + w.pair(x[i].w, z[i].w, v + 3);
      }
    }
    for (int v = b0 + (n4 << 2) + threadIdx.x; v < b1; v += SAMPLE_THREADS) sacc += w(v);
    const float sk = block_sum<SAMPLE_THREADS>(sacc, red);
    if (threadIdx.x == 0) {
      a.resid_part[(size_t)req * a.nch + k] = sk;
      __threadfence();
      const unsigned done = atomicAdd(&a.resid_counter[req], 1u);
      const bool last = (done == (unsigned)a.nch - 1);
      if (last) a.resid_counter[req] = 0u;
      s_last = last;
    }
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  int slot, pos0;
  uint32_t stream;
  verify_request_ctx(a, req, &slot, &pos0, &stream);
  const float u = philox_uniform(a.seed, stream, (uint32_t)(pos0 + at), KIND_RESID);
  const float* cs = a.resid_part + (size_t)req * a.nch;
  __shared__ float s_Z, s_base;
  __shared__ int s_k;
  if (threadIdx.x < 32) {
    // Z and the crossing chunk come from one chunk-order scan; the target
    // u * Z needs Z first, so the scan runs twice (the second only reads)
    const PartW pw{cs};
    const float Z = warp_chunk_pick(pw, a.nch, INFINITY).total;
    ChunkPick cp = warp_chunk_pick(pw, a.nch, u * Z);
    if (cp.k < 0) { cp.k = cp.lastk; cp.base = 0.f; }
    if (threadIdx.x == 0) { s_Z = Z; s_k = cp.k; s_base = cp.base; }
  }
  __syncthreads();
  const float Z = s_Z;
  int y;
  if (Z > 0.f && s_k >= 0) {
    int lastpos;
    const int b0 = s_k * a.ch, b1 = min(a.V, b0 + a.ch);
    y = chunk_crossing(w, b0, b1, s_base, u * Z, &lastpos, red);
    if (y < 0) y = lastpos >= 0 ? lastpos : b0;
  } else {
    // no residual mass after rounding: draw from p
    __shared__ RowStat s_rs;
    if (threadIdx.x < 32) {
      const RowStat rs = combine_row(a.partial + (rbase + at) * a.nch, a.nch);
      if (threadIdx.x == 0) s_rs = rs;
    }
    __syncthreads();
    y = sample_from_partials<FILT>(prow, a.partial + (rbase + at) * a.nch, a.nch, a.ch, a.V, s_rs, u,
                                   red, fp);
  }
  verify_finish(a, req, slot, pos0, at, y);
}


// ---------------------------------------------------------------------------
// Nucleus threshold of a row (top-p), one CTA per row.
//
// The masses are weights w_v = exp(l_v - max) as fixed-point integers
// (2^40 units, rounded): integer sums are exact whatever their order, so the
// result does not depend on scheduling.  A radix select over the 32-bit keys,
// eight bits per pass from the most significant, finds the key kappa of the
// token whose cumulative mass (most probable first) first reaches
// T = top_p * (total mass): each pass builds a mass histogram of the keys
// that share the prefix found so far (one histogram per warp, then added per
// bin), and one warp scans the bins from the highest.  Tokens with a key
// above kappa are kept; of the tokens whose logit is exactly kappa's, the
// first j by token id are kept, j the least count that reaches T.
// ---------------------------------------------------------------------------
constexpr int NUC_THREADS = 1024;
constexpr int NUC_WARPS = NUC_THREADS / 32;
constexpr int NUC_SMEM = NUC_WARPS * 256 * 8;          // per-warp histograms
constexpr float NUC_SCALE = 1099511627776.0f;           // 2^40

struct TopPArgs {
  const float* logits; int V;            // V % 4 == 0
  int rows_per_req;                      // rows filtered per request
  int64_t logit_rows_per_req;
  int draft_map;                         // 1: filtered row s is logit row (s == 0 ? 0 : s + 1)
  float top_p;                           // in (0, 1)
  RowFilter* out;                        // entry of each filtered logit row [n_req * logit_rows_per_req]
};

__device__ __forceinline__ unsigned long long nuc_weight(float l, float ML) {
  return __float2ull_rn(exp_rel(l, ML) * NUC_SCALE);
}

__global__ void __launch_bounds__(NUC_THREADS) top_p_kernel(const TopPArgs a) {
  extern __shared__ unsigned long long nuc_hist[];       // [NUC_WARPS][256]
  __shared__ float s_red[NUC_WARPS];
  __shared__ unsigned long long s_bin[256];
  __shared__ uint32_t s_prefix;
  __shared__ unsigned long long s_above, s_mass;
  __shared__ double s_T;
  __shared__ int s_need, s_ntied, s_cut;
  __shared__ int s_cnt[NUC_WARPS];
  pdl_trigger();
  pdl_wait();
  const int rid = blockIdx.x;
  const int req = rid / a.rows_per_req, srow = rid % a.rows_per_req;
  const int lrow = (a.draft_map && srow > 0) ? srow + 1 : srow;
  const size_t orow = (size_t)req * a.logit_rows_per_req + lrow;
  const float* row = a.logits + orow * a.V;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int n4 = a.V >> 2;

  // the row max
  float m = -INFINITY;
  for (int j = tid; j < n4; j += NUC_THREADS) {
    const float4 x = r4[j];
    m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
  }
  m = warp_max(m);
  if (lane == 0) s_red[wid] = m;
  __syncthreads();
  float M = s_red[0];
  for (int w = 1; w < NUC_WARPS; ++w) M = fmaxf(M, s_red[w]);
  const float ML = M * SAMPLE_LOG2E;

  unsigned long long* hist = nuc_hist + wid * 256;
  uint32_t prefix = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = lane; b < 256; b += 32) hist[b] = 0ull;
    __syncwarp();
    for (int j = tid; j < n4; j += NUC_THREADS) {
      const float4 x = r4[j];
      const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t k = logit_key(xs[e]);
        if (pass == 0 || (k >> (shift + 8)) == prefix) {
          const unsigned long long w = nuc_weight(xs[e], ML);
          if (w) atomicAdd(&hist[(k >> shift) & 255u], w);
        }
      }
    }
    __syncthreads();
    for (int b = tid; b < 256; b += NUC_THREADS) {
      unsigned long long t = 0;
      for (int w = 0; w < NUC_WARPS; ++w) t += nuc_hist[w * 256 + b];
      s_bin[b] = t;
    }
    __syncthreads();
    if (wid == 0) {
      // lane l holds bins 255 - 8 l - e, e = 0..7: keys in descending order
      unsigned long long bm[8], lsum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        bm[e] = s_bin[255 - 8 * lane - e];
        lsum += bm[e];
      }
      unsigned long long incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (pass == 0) {
        // T = top_p * total mass (every key is in range in the first pass)
        const unsigned long long tot = __shfl_sync(0xffffffffu, incl, 31);
        if (lane == 0) { s_T = (double)a.top_p * (double)tot; s_above = 0ull; }
        __syncwarp();
      }
      const double T = s_T;
      const unsigned long long above = s_above;
      __syncwarp();
      const unsigned hit = __ballot_sync(0xffffffffu, (double)(above + incl) >= T);
      const int hl = hit ? __ffs(hit) - 1 : 31;
      if (lane == hl) {
        unsigned long long run = above + (incl - lsum);
        int bsel = 255 - 8 * lane - 7;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if ((double)(run + bm[e]) >= T) { bsel = 255 - 8 * lane - e; break; }
          run += bm[e];
        }
        s_prefix = (prefix << 8) | (uint32_t)bsel;
        s_above = run;
        s_mass = s_bin[bsel];
      }
    }
    __syncthreads();
    prefix = s_prefix;
  }
  // the tokens whose logit is kappa's: how many, and how many are needed
  if (tid == 0) {
    const unsigned long long wk = nuc_weight(key_logit(prefix), ML);
    long long ntied = wk ? (long long)(s_mass / wk) : 1;
    if (ntied < 1) ntied = 1;
    long long need = wk ? (long long)ceil((s_T - (double)s_above) / (double)wk) : 1;
    need = need < 1 ? 1 : (need > ntied ? ntied : need);
    s_need = (int)need;
    s_ntied = (int)ntied;
    s_cut = a.V - 1;
  }
  __syncthreads();
  if (s_need < s_ntied) {
    // the need-th token (by id) with key kappa: thread-contiguous segments,
    // a block scan of the per-thread counts
    const int per = (a.V + NUC_THREADS - 1) / NUC_THREADS;
    const int b0 = tid * per, b1 = min(a.V, b0 + per);
    int cnt = 0;
    for (int v = b0; v < b1; ++v) cnt += logit_key(row[v]) == prefix;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_cnt[wid] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < wid; ++w) base += s_cnt[w];
    const int excl = base + incl - cnt;
    const int need = s_need;
    if (excl < need && excl + cnt >= need) {
      int c = excl;
      for (int v = b0; v < b1; ++v)
        if (logit_key(row[v]) == prefix && ++c == need) { s_cut = v; break; }
    }
    __syncthreads();
  }
  if (tid == 0) a.out[orow] = RowFilter{prefix, s_cut};
}

}  // namespace uno
