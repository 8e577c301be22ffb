// Tree sampler of the Psi-Spec iteration (per-request throughput at batch 1;
// summary page "通过离散扩散实现 LLM 无损加速：扩散增强自回归模型", section
// 方法关键点 names a linear and a tree sampler; the blog page's list of the two
// candidate-set modes is lost).  Reading, as in the CPU oracle: the block's
// first token x_1 comes from the AR row; k chains draw positions 2..B
// independently from the drafter's rows (chain j with Philox lane j, so chain
// 0 is the linear sampler's block); one verify pass scores every chain
// [x_1, y_j2, ..., y_jB]; the walk then applies recursive rejection at each
// position over its candidates - every chain's token at position 2; later,
// the continuing chain's token first, then the other chains' tokens, which
// end the block if accepted.  A rejection replaces the target r by
// max(0, r - q) renormalised; if every candidate is rejected the token is
// drawn from the last r.  With k = 1 this is the linear sampler.
//
// Kernels (decode step with the tree on):
//   row_lse_kernel     log-normaliser of each chain row of the verify pass;
//   tree_walk_kernel   one CTA per request: the walk, the emitted tokens and
//                      the request state (each full-vocabulary pass is a
//                      fixed-order block reduction or scan: deterministic);
//   tree_commit_kernel copies the accepted chain's keys/values (positions
//                      c+1 .. c+m) from its scratch slot into the request's
//                      slot.
#pragma once

#include <climits>

#include "layers.cuh"
#include "sampling.cuh"

namespace uno {

constexpr int TREE_THREADS = 1024;

// ---------------------------------------------------------------------------
// log-normaliser of rows (one CTA per row, two passes: max, then sum).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(TREE_THREADS) row_lse_kernel(const float* logits, int V,
                                                               float* lse) {
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const float* row = logits + (size_t)blockIdx.x * V;
  float m = -INFINITY;
  for (int v = threadIdx.x; v < V; v += TREE_THREADS) m = fmaxf(m, row[v]);
  const float M = block_max<TREE_THREADS>(m, red);
  const float ML = M * SAMPLE_LOG2E;
  float s = 0.f;
  for (int v = threadIdx.x; v < V; v += TREE_THREADS) s += exp_rel(row[v], ML);
  const float S = block_sum<TREE_THREADS>(s, red);
  if (threadIdx.x == 0) lse[blockIdx.x] = M + logf(S);
}

struct TreeArgs {
  const float* q;            // draft-pass logits [n_req, B+1, V] (row d: q of position c+d)
  const float* lse_q;        // [n_req, B]: lse of q row d at index d - 1
  const float* p;            // tree verify logits [n_req, k, B, V]: row i of chain j is
                             //   p of position c+2+i given chain j's tokens up to depth i+1
  const float* lse_p;        // [n_req, k, B]
  const int32_t* chains;     // [n_req, k, B]: x_1, y_j2 .. y_jB
  int V, B, k;
  uint64_t seed;
  const int32_t* req_slot; int32_t* cached; int32_t* pending; const uint32_t* slot_stream;
  float* resid;              // [n_req, 2, V] scratch (the residual target, ping-pong)
  int32_t* out_tok; int out_stride; int32_t* n_out;
  int32_t* walk;             // [n_req, 3]: c, m (accepted path length), chain of the path
  int32_t* status;
};

// Inverse CDF over w(v), v in [0, V) (whole CTA): thread-contiguous segments,
// a block scan of their sums, then the crossing inside the segment: the
// smallest v whose inclusive prefix exceeds u * (total); if rounding leaves
// none, the last v with w > 0.  The total comes from the same sums.
template <typename W>
__device__ int blk_inverse_cdf(const W& w, int V, float u, float* red) {
  __shared__ float s_tot[TREE_THREADS / 32];
  __shared__ int s_hit, s_last;
  const int per = (V + TREE_THREADS - 1) / TREE_THREADS;
  const int b0 = threadIdx.x * per, b1 = min(V, b0 + per);
  float ts = 0.f;
  int lastpos = -1;
  for (int v = b0; v < b1; ++v) {
    const float x = w(v);
    ts += x;
    if (x > 0.f) lastpos = v;
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  float incl = ts;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (threadIdx.x == 0) { s_hit = INT_MAX; s_last = -1; }
  if (lane == 31) s_tot[wid] = incl;
  __syncthreads();
  float base = 0.f, total = 0.f;
  for (int k = 0; k < TREE_THREADS / 32; ++k) {
    if (k < wid) base += s_tot[k];
    total += s_tot[k];
  }
  const float target = u * total;
  float run = base + (incl - ts);
  if (run + ts > target && b0 < b1) {
    for (int v = b0; v < b1; ++v) {
      run += w(v);
      if (run > target) { atomicMin(&s_hit, v); break; }
    }
  }
  if (lastpos >= 0) atomicMax(&s_last, lastpos);
  __syncthreads();
  const int hit = s_hit, last = s_last;
  __syncthreads();
  (void)red;
  return hit != INT_MAX ? hit : (last >= 0 ? last : 0);
}

struct SoftW {     // exp(l - lse): the row's probabilities
  const float* l; float lseL;
  __device__ __forceinline__ float operator()(int v) const { return exp_rel(l[v], lseL); }
};
struct BufW {      // an explicit weight row
  const float* r;
  __device__ __forceinline__ float operator()(int v) const { return r[v]; }
};

// One CTA per request.
__global__ void __launch_bounds__(TREE_THREADS) tree_walk_kernel(const TreeArgs a) {
  __shared__ float red[32];
  __shared__ int s_acc;
  pdl_trigger();
  pdl_wait();
  const int req = blockIdx.x, B = a.B, k = a.k, V = a.V;
  const int slot = a.req_slot[req];
  const int c = a.cached[slot];
  const uint32_t stream = a.slot_stream[slot];
  const int32_t* ch = a.chains + (size_t)req * k * B;
  float* R0 = a.resid + (size_t)req * 2 * V;
  int path[64];          // accepted tokens along the continuing chain (B <= 64)
  int m = 1, jstar = -1, last = -1;
  path[0] = ch[0];
  bool done = false;
  for (int d = 2; d <= B && !done; ++d) {
    const int pj = d == 2 ? 0 : jstar, pi = d == 2 ? 0 : d - 2;
    const float* pl = a.p + (((size_t)req * k + pj) * B + pi) * V;
    const float lse_p = a.lse_p[((size_t)req * k + pj) * B + pi];
    const float* ql = a.q + ((size_t)req * (B + 1) + d) * V;
    const float lse_q = a.lse_q[(size_t)req * B + d - 1];
    const float lpL = lse_p * SAMPLE_LOG2E, lqL = lse_q * SAMPLE_LOG2E;
    // the target r: p itself (cur = -1) or the residual row R0 + cur V over Z
    int cur = -1;
    float invZ = 1.f;
    int acc = -1, acc_j = -1;
    for (int t = 0; t < k; ++t) {
      const int j = d == 2 ? t : (t == 0 ? jstar : (t <= jstar ? t - 1 : t));
      const int y = ch[j * B + d - 1];
      if (threadIdx.x == 0) {
        const float u = philox_uniform(a.seed, stream, (uint32_t)(c + d), KIND_ACCEPT, (uint32_t)j);
        bool ok;
        if (y < 0 || y >= V) { raise_status(a.status, ST_BAD_TOKEN); ok = false; }
        else if (cur < 0) ok = logf(u) < (pl[y] - lse_p) - (ql[y] - lse_q);
        else {
          const float rv = R0[(size_t)cur * V + y] * invZ;
          ok = rv > 0.f && logf(u) < logf(rv) - (ql[y] - lse_q);
        }
        s_acc = ok ? 1 : 0;
      }
      __syncthreads();
      const bool ok = s_acc != 0;
      __syncthreads();
      if (ok) { acc = y; acc_j = j; break; }
      // rejected: r <- max(0, r - q), renormalised (kept if it has no mass)
      const int nxt = cur < 0 ? 0 : 1 - cur;
      float* Rn = R0 + (size_t)nxt * V;
      const float* Rc = R0 + (size_t)(cur < 0 ? 0 : cur) * V;
      float zs = 0.f;
      for (int v = threadIdx.x; v < V; v += TREE_THREADS) {
        const float rv = cur < 0 ? exp_rel(pl[v], lpL) : Rc[v] * invZ;
        const float x = fmaxf(rv - exp_rel(ql[v], lqL), 0.f);
        Rn[v] = x;
        zs += x;
      }
      const float Z = block_sum<TREE_THREADS>(zs, red);
      if (Z > 0.f) { cur = nxt; invZ = 1.f / Z; }
      __syncthreads();
    }
    if (acc >= 0) {
      if (d == 2 || acc_j == jstar) {
        jstar = acc_j;
        path[m++] = acc;
        continue;
      }
      last = acc;                 // another chain's token: the block ends with it
      done = true;
      break;
    }
    // every candidate rejected: draw from the last target
    const float u = philox_uniform(a.seed, stream, (uint32_t)(c + d), KIND_RESID, 0u);
    last = cur < 0 ? blk_inverse_cdf(SoftW{pl, lpL}, V, u, red)
                   : blk_inverse_cdf(BufW{R0 + (size_t)cur * V}, V, u, red);
    done = true;
  }
  if (!done) {
    // the continuing chain was accepted to position B: the bonus token
    const float* pl = a.p + (((size_t)req * k + jstar) * B + (B - 1)) * V;
    const float lse_p = a.lse_p[((size_t)req * k + jstar) * B + (B - 1)];
    const float u = philox_uniform(a.seed, stream, (uint32_t)(c + B + 1), KIND_RESID, 0u);
    last = blk_inverse_cdf(SoftW{pl, lse_p * SAMPLE_LOG2E}, V, u, red);
  }
  if (threadIdx.x == 0) {
    int32_t* out = a.out_tok + (size_t)req * a.out_stride;
    for (int i = 0; i < m; ++i) out[i] = path[i];
    out[m] = last;
    a.n_out[req] = m + 1;
    a.walk[(size_t)req * 3 + 0] = c;
    a.walk[(size_t)req * 3 + 1] = m;
    a.walk[(size_t)req * 3 + 2] = jstar < 0 ? 0 : jstar;
    a.cached[slot] = c + m + 1;
    a.pending[slot] = last;
  }
}

// Keys/values of the accepted path: positions c+1 .. c+m of the path's chain
// slot into the request's slot.  Grid (B, n_layers, n_req); positions past m
// exit.  Chain slot of (request slot r, chain j): max_batch + r TREE_MAX_K + j.
struct TreeCommitArgs {
  KvLayout kv;
  int max_batch, esz;
  const int32_t* req_slot;
  const int32_t* walk;
  int32_t* status;
};
__global__ void __launch_bounds__(256) tree_commit_kernel(const TreeCommitArgs a) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x + 1, layer = blockIdx.y, req = blockIdx.z;
  const int c = a.walk[(size_t)req * 3], m = a.walk[(size_t)req * 3 + 1], j = a.walk[(size_t)req * 3 + 2];
  if (i > m) return;
  const int slot = a.req_slot[req];
  const int cs = a.max_batch + slot * TREE_MAX_K + j;
  const int pos = c + i;
  int ok_s, ok_d;
  const int ps = a.kv.page_of(cs, pos, ok_s), pd = a.kv.page_of(slot, pos, ok_d);
  if (!ok_s || !ok_d) {
    if (threadIdx.x == 0) raise_status(a.status, ST_POS_OVERFLOW);
    return;
  }
  // per plane and head, head_dim contiguous elements: copied as 4-byte words
  const int words = a.kv.head_dim * a.esz / 4;
  const int n = a.kv.n_planes * a.kv.n_kv_heads * words;
  const uint32_t* src = reinterpret_cast<const uint32_t*>(a.kv.pool);
  uint32_t* dst = reinterpret_cast<uint32_t*>(a.kv.pool);
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int w = e % words, hp = e / words;
    const int head = hp % a.kv.n_kv_heads, plane = hp / a.kv.n_kv_heads;
    const size_t so = a.kv.offset_in_page(layer, ps, pos, plane, head) * a.esz / 4 + w;
    const size_t doff = a.kv.offset_in_page(layer, pd, pos, plane, head) * a.esz / 4 + w;
    dst[doff] = src[so];
  }
}

}  // namespace uno
