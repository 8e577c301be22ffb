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
// Inverse-CDF sampling on the device: w_v = expf(l_v - M) with M the row max;
// Z = sum over chunks (in chunk order) of s_k * expf(m_k - M); the token is in
// the first chunk whose running prefix exceeds u * Z, at the first element
// whose within-chunk inclusive prefix (thread-contiguous order, fixed) pushes
// the running sum above u * Z.  When rounding leaves no crossing, the last
// element with positive weight (of the chunk, or of the row) is taken.
#pragma once

#include <climits>

#include "common.cuh"

namespace uno {

constexpr int SAMPLE_THREADS = 256;

// ---------------------------------------------------------------------------
// Phase A: reduce one chunk of one row to (max, sum exp(l - max)).  Each
// thread reduces its own logits to a (max, sum) pair; the pairs are combined
// across the CTA in a fixed tree (warp butterfly, then the warps in order),
// so one reduction serves both statistics.
// ---------------------------------------------------------------------------
constexpr int CHUNK_IT = 8;   // float4 per thread: a chunk holds <= 8 * 4 * 256 = 8192 logits
__device__ __forceinline__ float2 ms_combine(float2 a, float2 b) {
  const float M = fmaxf(a.x, b.x);
  if (M == -INFINITY) return make_float2(M, 0.f);
  return make_float2(M, a.y * expf(a.x - M) + b.y * expf(b.x - M));
}
__device__ __forceinline__ float2 reduce_chunk(const float* row, int c0, int c1, float* red) {
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
  float s = 0.f;
  if (m != -INFINITY) {
#pragma unroll
    for (int i = 0; i < CHUNK_IT; ++i) {
      const int j = threadIdx.x + i * SAMPLE_THREADS;
      if (j < n4) s += expf(v[i].x - m) + expf(v[i].y - m) + expf(v[i].z - m) + expf(v[i].w - m);
    }
    for (int j = c0 + (n4 << 2) + threadIdx.x; j < c1; j += SAMPLE_THREADS) s += expf(row[j] - m);
  }
  float2 ms = make_float2(m, s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    ms = ms_combine(ms, make_float2(__shfl_xor_sync(0xffffffffu, ms.x, o),
                                    __shfl_xor_sync(0xffffffffu, ms.y, o)));
  float2* red2 = reinterpret_cast<float2*>(red);     // SAMPLE_THREADS / 32 pairs
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  __syncthreads();                                    // red may hold a previous reduction
  if (lane == 0) red2[wid] = ms;
  __syncthreads();
  float2 t = red2[0];
#pragma unroll
  for (int w = 1; w < SAMPLE_THREADS / 32; ++w) t = ms_combine(t, red2[w]);
  return t;
}

// Row-level combine of chunk pairs (run by one thread, chunk order).
struct RowStat { float M, Z; };
__device__ __forceinline__ RowStat combine_row(const float2* part, int nch) {
  float M = -INFINITY;
  for (int k = 0; k < nch; ++k) M = fmaxf(M, __ldcg(&part[k].x));
  float Z = 0.f;
  for (int k = 0; k < nch; ++k) {
    const float2 pk = __ldcg(&part[k]);
    if (pk.x != -INFINITY) Z += pk.y * expf(pk.x - M);
  }
  return {M, Z};
}

// Weight functors used by the crossing scan (get4: four weights from v, a
// multiple of 4).
struct SoftmaxW {
  const float* row; float M;
  __device__ __forceinline__ float operator()(int v) const { return expf(row[v] - M); }
  __device__ __forceinline__ void get4(int v, float* w) const {
    const float4 x = *reinterpret_cast<const float4*>(row + v);
    w[0] = expf(x.x - M); w[1] = expf(x.y - M); w[2] = expf(x.z - M); w[3] = expf(x.w - M);
  }
};
struct ResidW {
  const float* p; const float* q; float lse_p, lse_q;
  __device__ __forceinline__ float pair(float pv, float qv) const {
    const float d = expf(pv - lse_p) - expf(qv - lse_q);
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
  __shared__ int s_lastk;
  const float target = u * rs.Z;
  if (threadIdx.x == 0) {
    float run = 0.f;
    int kk = -1, lastk = -1;
    for (int k = 0; k < nch; ++k) {
      const float2 pk = __ldcg(&part[k]);
      const float sk = (pk.x != -INFINITY) ? pk.y * expf(pk.x - rs.M) : 0.f;
      if (sk > 0.f) lastk = k;
      if (kk < 0 && run + sk > target) { kk = k; s_base = run; }
      run += sk;
    }
    if (kk < 0) { kk = lastk; s_base = 0.f; }
    s_k = kk;
    s_lastk = lastk;
  }
  __syncthreads();
  const int k = s_k;
  const float base = s_base;
  __syncthreads();
  if (k < 0) return 0;  // empty row (all -inf): only reachable with invalid logits
  SoftmaxW w{row, rs.M};
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
  if (threadIdx.x == 0) s_rs = combine_row(part, a.nch);
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

__global__ void __launch_bounds__(SAMPLE_THREADS, 3) spec_verify_kernel(const VerifyArgs a) {
  __shared__ float red[32];
  __shared__ bool s_last;
  __shared__ int s_a;
  pdl_trigger();
  pdl_wait();
  const int k = blockIdx.x;
  const int rid = blockIdx.y;
  const int req = rid / a.rows_red, r = rid % a.rows_red;
  const float* row;
  if (r < a.n_p) {
    const int br = (r < a.n_tests) ? a.p_row0 + r : a.bonus_row;
    row = a.p + ((size_t)req * a.p_req_rows + br) * a.V;
  } else {
    row = a.q + ((size_t)req * a.q_req_rows + a.q_row0 + (r - a.n_p)) * a.V;
  }
  const int c0 = k * a.ch, c1 = min(a.V, c0 + a.ch);
  const float2 pr = reduce_chunk(row, c0, c1, red);
  if (threadIdx.x == 0) {
    a.partial[(size_t)rid * a.nch + k] = pr;
    __threadfence();
    const unsigned done = atomicAdd(&a.row_counter[rid], 1u);
    bool last = (done == (unsigned)a.nch - 1);
    if (last) {
      a.row_counter[rid] = 0u;
      const RowStat rs = combine_row(a.partial + (size_t)rid * a.nch, a.nch);
      a.lse[rid] = rs.M + logf(rs.Z);
      __threadfence();
      const unsigned rdone = atomicAdd(&a.req_counter[req], 1u);
      last = (rdone == (unsigned)a.rows_red - 1);
      if (last) a.req_counter[req] = 0u;
    }
    s_last = last;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- request decision (one CTA per request) ----
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
  const int at = s_a;   // accepted prefix length among the tests
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
    if (threadIdx.x == 0) s_rs2 = combine_row(a.partial + (rbase + a.n_tests) * a.nch, a.nch);
    __syncthreads();
    y = sample_from_partials(prow, a.partial + (rbase + a.n_tests) * a.nch, a.nch, a.ch, a.V,
                             s_rs2, u, red);
  }
  if (threadIdx.x == 0) a.at_ws[req] = -1;
  verify_finish(a, req, slot, pos0, at, y);
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
  const ResidW w{prow, qrow, lse_p, lse_q};
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
  if (threadIdx.x == 0) {
    float Z = 0.f;
    for (int c = 0; c < a.nch; ++c) Z += __ldcg(&cs[c]);
    const float target = u * Z;
    float run = 0.f;
    int kk = -1, lastk = -1;
    float base = 0.f;
    for (int c = 0; c < a.nch; ++c) {
      const float sk = __ldcg(&cs[c]);
      if (sk > 0.f) lastk = c;
      if (kk < 0 && run + sk > target) { kk = c; base = run; }
      run += sk;
    }
    if (kk < 0) { kk = lastk; base = 0.f; }
    s_Z = Z;
    s_k = kk;
    s_base = base;
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
    if (threadIdx.x == 0) s_rs = combine_row(a.partial + (rbase + at) * a.nch, a.nch);
    __syncthreads();
    y = sample_from_partials(prow, a.partial + (rbase + at) * a.nch, a.nch, a.ch, a.V, s_rs, u, red);
  }
  verify_finish(a, req, slot, pos0, at, y);
}

}  // namespace uno
