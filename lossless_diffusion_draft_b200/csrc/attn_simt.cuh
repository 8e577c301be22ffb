// Paged-KV grouped-query attention with the block-causal mask, SIMT form
// (fp32 models, prefill, and any shape the tensor-core kernel does not take).
//
// Mask (blog page "…Uno 的无损加速之路", section Diffusion Distillation：一步蒸馏 +
// 块级扩散): the clean sequence is causal; a noised block is causal inside
// itself and sees every clean token before it.  A row's keys are the two
// ranges of RowKeys (layers.cuh).  In a decode pass the keys are [cache
// 0..c-1, pending c, block c+1..c+B] of one slot, all written to the pool by
// the RoPE/KV kernel before this one runs, and the rule reduces to "key
// position <= query position" for every row of both passes.
//
// One CTA takes (split s, query tile, request x kv head): up to 72 query rows
// (tokens x the kv head's query heads), streams its share of the key range in
// tiles of 32 keys through shared memory, and keeps an online softmax per
// query row.  With several splits, each CTA writes (m, l, o) partials and the
// last CTA of the group (atomic counter, no waiting) merges them in split
// order.
#pragma once

#include "common.cuh"
#include "layers.cuh"

namespace uno {

constexpr int ATT_THREADS = 128;
constexpr int ATT_MAXQ = 72;     // query rows per CTA
constexpr int ATT_KT = 32;       // keys per tile

struct AttnParams {
  const void* qkv; int ld_qkv;   // rotated q in columns [0, H*hd)
  const void* q_lo;              // its rounding residual rows (same layout), or null
  void* out; int ld_out;         // [M, H*hd]
  void* out_lo;                  // rounding residual rows (split GEMM input) or null
  KvLayout kv; int layer;
  int H, Hkv;
  float scale;
  int rows_per_req;
  const int32_t* row_pos; const int32_t* row_slot;
  RowKeys keys;                   // per-row key ranges (block-causal rule)
  int n_splits, n_qtiles;
  float* ws; unsigned* counters;  // split partials, per-group counters (zero, left zero)
};

template <typename T, int HD>
__global__ void __launch_bounds__(ATT_THREADS) attn_simt_kernel(const AttnParams p) {
  constexpr int EPL = (HD + 31) / 32;
  constexpr int QPW = ATT_MAXQ / (ATT_THREADS / 32);   // query rows per warp
  extern __shared__ float sm[];
  float* q_s = sm;                                   // [ATT_MAXQ][HD]
  float* k_s = q_s + ATT_MAXQ * HD;                  // [KT][HD + 1]
  float* v_s = k_s + ATT_KT * (HD + 1);              // [KT][HD]
  __shared__ bool s_last;
  pdl_trigger();
  pdl_wait();

  const int split = blockIdx.x, qt = blockIdx.y, z = blockIdx.z;
  const int req = z / p.Hkv, kvh = z % p.Hkv;
  const int G = p.H / p.Hkv;
  const int TQ = ATT_MAXQ / G;
  const int tok0 = qt * TQ;
  const int ntok = min(TQ, p.rows_per_req - tok0);
  if (ntok <= 0) return;
  const int nq = ntok * G;
  const int row0 = req * p.rows_per_req + tok0;
  // the tile list: key tiles of the clean range, then of the noised range
  const KeyTiles kt = p.keys.tiles(p.row_pos, p.row_slot, row0, ntok, ATT_KT,
                                   p.kv.pages_per_req * (KV_PAGE / ATT_KT));
  const int ntiles = kt.n1 + kt.n2;
  const int t_begin = (int)((long long)ntiles * split / p.n_splits);
  const int t_end = (int)((long long)ntiles * (split + 1) / p.n_splits);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  typedef typename KvOf<T>::type KV;   // q and the KV cache
  const KV* qkv = reinterpret_cast<const KV*>(p.qkv);
  for (int idx = threadIdx.x; idx < nq * HD; idx += ATT_THREADS) {
    const int qi = idx / HD, d = idx % HD;
    const int tk = qi / G, g = qi % G;
    const size_t e = (size_t)(row0 + tk) * p.ld_qkv + (size_t)(kvh * G + g) * HD + d;
    const float qlo = p.q_lo ? to_f(reinterpret_cast<const KV*>(p.q_lo)[e]) : 0.f;
    q_s[idx] = (to_f(qkv[e]) + qlo) * p.scale;
  }
  float m_i[QPW], l_i[QPW], o_i[QPW][EPL];
  int qlim[QPW], qlo2[QPW], qhi2[QPW];   // each row's clean range [0, lim), noised [lo2, hi2)
#pragma unroll
  for (int t = 0; t < QPW; ++t) {
    m_i[t] = -INFINITY; l_i[t] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o_i[t][e] = 0.f;
    const int qi = warp + 4 * t;
    qlim[t] = qlo2[t] = qhi2[t] = 0;
    if (qi < nq) p.keys.ranges(p.row_pos, row0 + qi / G, qlim[t], qlo2[t], qhi2[t]);
  }

  const KV* pool = reinterpret_cast<const KV*>(p.kv.pool);
  for (int tile = t_begin; tile < t_end; ++tile) {
    const bool seg2 = tile >= kt.n1;
    const int kp0 = (seg2 ? kt.p2 + (tile - kt.n1) : tile) * ATT_KT;
    const int tslot = seg2 ? kt.slot2 : kt.slot1;
    __syncthreads();
    for (int idx = threadIdx.x; idx < ATT_KT * HD; idx += ATT_THREADS) {
      const int j = idx / HD, d = idx % HD;
      const int kp = kp0 + j;
      float kval = 0.f, vval = 0.f;
      {
        int ok;
        const size_t off = p.kv.offset(p.layer, tslot, kp, 0, kvh, ok);
        if (ok) {
          kval = to_f(pool[off + d]);
          if (p.kv.n_planes == 3) kval += to_f(pool[off + p.kv.plane_stride() + d]);   // K lo
          vval = to_f(pool[off + p.kv.v_plane() * p.kv.plane_stride() + d]);
        }
      }
      k_s[j * (HD + 1) + d] = kval;
      v_s[j * HD + d] = vval;
    }
    __syncthreads();
    const int kp = kp0 + lane;
#pragma unroll
    for (int t = 0; t < QPW; ++t) {
      const int qi = warp + 4 * t;
      if (qi >= nq) continue;
      float sc = -INFINITY;
      if (seg2 ? (kp >= qlo2[t] && kp < qhi2[t]) : kp < qlim[t]) {
        float dot = 0.f;
        const float* qr = q_s + qi * HD;
        const float* kr = k_s + lane * (HD + 1);
#pragma unroll 16
        for (int d = 0; d < HD; ++d) dot = fmaf(qr[d], kr[d], dot);
        sc = dot;
      }
      const float mx = warp_max(sc);
      const float m_new = fmaxf(m_i[t], mx);
      if (m_new == -INFINITY) continue;
      const float pj = (sc == -INFINITY) ? 0.f : expf(sc - m_new);
      const float corr = (m_i[t] == -INFINITY) ? 0.f : expf(m_i[t] - m_new);
      l_i[t] = l_i[t] * corr + warp_sum(pj);
#pragma unroll
      for (int e = 0; e < EPL; ++e) o_i[t][e] *= corr;
#pragma unroll 8
      for (int j = 0; j < ATT_KT; ++j) {
        const float pb = __shfl_sync(0xffffffffu, pj, j);
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const int d = lane + 32 * e;
          if (d < HD) o_i[t][e] = fmaf(pb, v_s[j * HD + d], o_i[t][e]);
        }
      }
      m_i[t] = m_new;
    }
  }

  T* out = reinterpret_cast<T*>(p.out);
  if (p.n_splits == 1) {
#pragma unroll
    for (int t = 0; t < QPW; ++t) {
      const int qi = warp + 4 * t;
      if (qi >= nq) continue;
      const float inv = 1.f / l_i[t];
      const int tk = qi / G, g = qi % G;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int d = lane + 32 * e;
        if (d < HD)
          store_split<T>(out, reinterpret_cast<T*>(p.out_lo),
                         (size_t)(row0 + tk) * p.ld_out + (size_t)(kvh * G + g) * HD + d, o_i[t][e] * inv);
      }
    }
    return;
  }
  // split partials: ws[group][split][q][HD + 2]
  const size_t group = (size_t)z * p.n_qtiles + qt;
  float* ws = p.ws + (group * p.n_splits + split) * ATT_MAXQ * (HD + 2);
#pragma unroll
  for (int t = 0; t < QPW; ++t) {
    const int qi = warp + 4 * t;
    if (qi >= nq) continue;
    float* w = ws + qi * (HD + 2);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int d = lane + 32 * e;
      if (d < HD) w[d] = o_i[t][e];
    }
    if (lane == 0) { w[HD] = m_i[t]; w[HD + 1] = l_i[t]; }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned done = atomicAdd(&p.counters[group], 1u);
    s_last = (done == (unsigned)p.n_splits - 1);
    if (s_last) p.counters[group] = 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* wg = p.ws + group * p.n_splits * ATT_MAXQ * (HD + 2);
  for (int idx = threadIdx.x; idx < nq * HD; idx += ATT_THREADS) {
    const int qi = idx / HD, d = idx % HD;
    float M = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s) M = fmaxf(M, __ldcg(wg + ((size_t)s * ATT_MAXQ + qi) * (HD + 2) + HD));
    float L = 0.f, O = 0.f;
    for (int s = 0; s < p.n_splits; ++s) {
      const float* w = wg + ((size_t)s * ATT_MAXQ + qi) * (HD + 2);
      const float ms = __ldcg(w + HD);
      if (ms == -INFINITY) continue;
      const float f = expf(ms - M);
      L += __ldcg(w + HD + 1) * f;
      O += __ldcg(w + d) * f;
    }
    const int tk = qi / G, g = qi % G;
    store_split<T>(out, reinterpret_cast<T*>(p.out_lo),
                   (size_t)(row0 + tk) * p.ld_out + (size_t)(kvh * G + g) * HD + d, O / L);
  }
}

}  // namespace uno
