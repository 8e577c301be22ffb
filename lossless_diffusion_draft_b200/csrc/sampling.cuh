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
// Phase A: reduce one chunk of one row to (max, sum exp(l - max)).  The
// CTA's max comes first (warp butterfly, then the warps' maxima in order),
// then every logit takes one exponential against it and the sums are added
// by a butterfly and the warps in order: a fixed tree, and no rescaling.
// ---------------------------------------------------------------------------
constexpr int CHUNK_IT = 8;   // float4 per thread: a chunk holds <= 8 * 4 * 256 = 8192 logits
// red: at least 2 * SAMPLE_THREADS / 32 floats of shared memory.
__device__ __forceinline__ float2 reduce_chunk(const float* row, int c0, int c1, float* red) {
  constexpr int NW = SAMPLE_THREADS / 32;
  // float4 path: rows start on 16-byte boundaries (vocab % 4 == 0 is required)
  const int n4 = (c1 - c0) >> 2;
  const float4* r4 = reinterpret_cast<const float4*>(row + c0);
  float4 v[CHUNK_IT];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < CHUNK_IT; ++i) {
    const int j = threadIdx.x + i * SAMPLE_THREADS;
    if (j < n4) {
      v[i] = __ldcs(r4 + j);
      m = fmaxf(m, fmaxf(fmaxf(v[i].x, v[i].y), fmaxf(v[i].z, v[i].w)));
    }
  }
  // scalar tail (chunk length not a multiple of 4: only the row's last chunk)
  for (int j = c0 + (n4 << 2) + threadIdx.x; j < c1; j += SAMPLE_THREADS) m = fmaxf(m, row[j]);
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
    for (int j = c0 + (n4 << 2) + threadIdx.x; j < c1; j += SAMPLE_THREADS) s += exp_rel(row[j], mL);
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
struct SoftmaxW {
  const float* row; float ML;          // row max x log2 e
  __device__ __forceinline__ float operator()(int v) const { return exp_rel(row[v], ML); }
  __device__ __forceinline__ void get4(int v, float* w) const {
    const float4 x = *reinterpret_cast<const float4*>(row + v);
    w[0] = exp_rel(x.x, ML); w[1] = exp_rel(x.y, ML); w[2] = exp_rel(x.z, ML); w[3] = exp_rel(x.w, ML);
  }
};
struct ResidW {
  const float* p; const float* q; float lpL, lqL;   // lse_p, lse_q x log2 e
  __device__ __forceinline__ float pair(float pv, float qv) const {
    const float d = exp_rel(pv, lpL) - exp_rel(qv, lqL);
    return d > 0.f ? d : 0.f;
  }
  __device__ __forceinline__ float operator()(int v) const { return pair(p[v], q[v]); }
  __device__ __forceinline__ void get4(int v, float* w) const {
    const float4 x = *reinterpret_cast<const float4*>(p + v);
    const float4 y = *reinterpret_cast<const float4*>(q + v);
    w[0] = pair(x.x, y.x); w[1] = pair(x.y, y.y); w[2] = pair(x.z, y.z); w[3] = pair(x.w, y.w);
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
__device__ int sample_from_partials(const float* row, const float2* part, int nch, int ch, int V,
                                    const RowStat& rs, float u, float* red) {
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
  SoftmaxW w{row, rs.M * SAMPLE_LOG2E};
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
};

__global__ void __launch_bounds__(SAMPLE_THREADS, 3) sample_rows_kernel(const SampleArgs a) {
  __shared__ float red[32];
  __shared__ bool s_last;
  pdl_trigger();
  pdl_wait();
  const int k = blockIdx.x;
  const int rid = blockIdx.y;
  const int req = rid / a.rows_per_req, s = rid % a.rows_per_req;
  const int lrow = (a.ar_mode || s == 0) ? 0 : s + 1;
  const float* row = a.logits + ((size_t)req * a.logit_rows_per_req + lrow) * a.V;
  const int c0 = k * a.ch, c1 = min(a.V, c0 + a.ch);
  const float2 pr = reduce_chunk(row, c0, c1, red);
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
  const int slot = a.req_slot[req];
  const int c = a.cached[slot];
  const uint32_t kind = (a.ar_mode || s == 0) ? KIND_FIRST : KIND_DRAFT;
  const float u = philox_uniform(a.seed, a.slot_stream[slot], (uint32_t)(c + 1 + s), kind);
  const int t = sample_from_partials(row, part, a.nch, a.ch, a.V, rs, u, red);
  if (threadIdx.x == 0) {
    if (a.ar_mode) {
      a.out_tok[req] = t;
      a.cached[slot] = c + 1;
      a.pending[slot] = t;
    } else {
      a.out_tok[(size_t)req * a.out_stride + s] = t;
      if (a.lse_out) a.lse_out[(size_t)req * a.rows_per_req + s] = rs.M + logf(rs.Z);
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
};

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
  return a.lse_q_in ? a.lse_q_in[(size_t)req * a.lse_q_stride + a.lse_q_off + j]
                    : __ldcg(&a.lse[(size_t)req * a.rows_red + a.n_p + j]);
}

// Outputs and commit of a request with `at` accepted tests and final token y
// (whole CTA).
__device__ void verify_finish(const VerifyArgs& a, int req, int slot, int pos0, int at, int y) {
  const bool decode = a.req_slot != nullptr;
  const int lead = decode ? 1 : 0;    // decode mode emits x_1 first
  int32_t* out = a.out_tok + (size_t)req * a.out_stride;
  for (int j = threadIdx.x; j < at; j += SAMPLE_THREADS)
    out[lead + j] = a.drafts[(size_t)req * a.drafts_stride + a.drafts_off + j];
  if (threadIdx.x == 0) {
    if (decode) {
      // emitted: x_1, the accepted x_2..x_{1+at}, then y; the cache grows by
      // n tokens (positions c..c+n-1 hold keys/values) and y becomes pending
      out[0] = a.first_tok[(size_t)req * a.drafts_stride];
      const int n = lead + at + 1;
      out[n - 1] = y;
      a.n_out[req] = n;
      a.cached[slot] = pos0 - 2 + n;
      a.pending[slot] = y;
    } else {
      out[at] = y;          // -1 when every test passed and no bonus row exists
      a.n_out[req] = at;
    }
  }
}

// The decision of request req once every reduced row's lse is in a.lse
// (whole CTA): the accept tests, the first rejection, and either the bonus
// draw and the commit here or the hand-over to spec_resid_kernel.
__device__ void verify_decide(const VerifyArgs& a, int req, float* red) {
  __shared__ int s_a;
  const size_t rbase = (size_t)req * a.rows_red;
  int slot, pos0;
  uint32_t stream;
  verify_request_ctx(a, req, &slot, &pos0, &stream);
  if (threadIdx.x == 0) s_a = a.n_tests;
  __syncthreads();
  for (int j = threadIdx.x; j < a.n_tests; j += SAMPLE_THREADS) {
    int t = a.drafts[(size_t)req * a.drafts_stride + a.drafts_off + j];
    if (t < 0 || t >= a.V) { raise_status(a.status, ST_BAD_TOKEN); t = 0; }
    const float* prow = a.p + ((size_t)req * a.p_req_rows + a.p_row0 + j) * a.V;
    const float* qrow = a.q + ((size_t)req * a.q_req_rows + a.q_row0 + j) * a.V;
    const float lse_p = __ldcg(&a.lse[rbase + j]);
    const float lse_q = verify_lse_q(a, req, j);
    const float u = philox_uniform(a.seed, stream, (uint32_t)(pos0 + j), KIND_ACCEPT);
    const bool acc = logf(u) < (prow[t] - lse_p) - (qrow[t] - lse_q);
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
    y = sample_from_partials(prow, a.partial + (rbase + a.n_tests) * a.nch, a.nch, a.ch, a.V,
                             s_rs2, u, red);
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
  return a.q + ((size_t)req * a.q_req_rows + a.q_row0 + (r - a.n_p)) * a.V;
}

// Fused form (few rows): grid (nch, n_req * rows_red).  The last chunk CTA
// of a row forms its lse, the last row of a request decides.
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
  const float2 pr = reduce_chunk(row, c0, c1, red);
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
  verify_decide(a, req, red);
}

// Split form (many rows), first kernel: grid (nch, n_req * rows_red), every
// CTA reduces its chunk, writes the pair and exits (no counters, no waiting
// on a round trip), so the loads of the next CTAs keep HBM busy.
__global__ void __launch_bounds__(SAMPLE_THREADS, 4) spec_reduce_kernel(const VerifyArgs a) {
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const int k = blockIdx.x;
  const int rid = blockIdx.y;
  const float* row = verify_row(a, rid / a.rows_red, rid % a.rows_red);
  const int c0 = k * a.ch, c1 = min(a.V, c0 + a.ch);
  const float2 pr = reduce_chunk(row, c0, c1, red);
  if (threadIdx.x == 0) a.partial[(size_t)rid * a.nch + k] = pr;
}

// Split form, second kernel: one CTA per request; warp w forms the lse of
// rows w, w + 8, ... (the same chunk-order combine as the fused form), then
// the CTA decides.
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
  verify_decide(a, req, red);
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
  const float* qrow = a.q + ((size_t)req * a.q_req_rows + a.q_row0 + at) * a.V;
  const float lse_p = __ldcg(&a.lse[rbase + at]);
  const float lse_q = verify_lse_q(a, req, at);
  const ResidW w{prow, qrow, lse_p * SAMPLE_LOG2E, lse_q * SAMPLE_LOG2E};
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
        if (j < n4) sacc += w.pair(x[i].x, z[i].x) + w.pair(x[i].y, z[i].y) +
                            w.pair(x[i].z, z[i].z) + w.pair(x[i].w, z[i].w);
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
    y = sample_from_partials(prow, a.partial + (rbase + at) * a.nch, a.nch, a.ch, a.V, s_rs, u, red);
  }
  verify_finish(a, req, slot, pos0, at, y);
}

}  // namespace uno
