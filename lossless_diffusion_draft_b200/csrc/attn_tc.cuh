// Paged-KV grouped-query attention with the block-causal mask on the
// 5th-generation tensor cores (fp16 q, K, V and P; fp32 scores, softmax and
// accumulators).
//
// Mask (blog page "不砸掉重来，给自回归 LLM 装一对“扩散翅膀”：Uno 的无损加速之路",
// section Diffusion Distillation：一步蒸馏 + 块级扩散): the clean sequence is
// causal; a noised block is causal inside itself and sees every clean token
// before it.  A row's keys are two ranges (RowKeys in layers.cuh): clean keys
// of its clean slot at positions [0, lim), and, for a noised row of the
// training form [x, z], noised keys of its own slot at [block start, pos].
// In the decode passes every key of a request (cache, pending token, block)
// is in its one slot and the rule is "key position <= query position".
//
// One CTA takes (key split, query tile, request x kv head).  Its 128 query
// rows are (token, head of the kv group) pairs, so the GQA group shares each
// K/V tile: 17 draft rows x 4 heads = 68 rows per KV stream.
//   warp 4  TMA: one KV page (64 keys) per tile, K and V as 64x64 boxes of the
//           pool viewed as a 2-D [rows, head_dim] tensor;
//   warp 5  MMA: S = Q K^T (M=128, N=64) into a double-buffered TMEM score
//           tile; O += P V (M=128, N=head_dim, B operand MN-major) into one
//           TMEM accumulator for the whole key range;
//   warps 0-3 (thread = query row): read the score row, softmax in the log2
//           domain against a reference max that moves (rescaling O in TMEM)
//           only when a tile's max exceeds it by more than 2^8, and write P
//           (fp16) to shared memory in the MMA's swizzled layout.
// With several key splits each CTA writes (m, l, O) partials and
// attn_merge_kernel (ATC_MERGE_ROWS query rows per CTA) adds them in split
// order.  Every wait is bounded.  While it runs, idle lanes of the producer
// warp prefetch the next projection's weights into L2.
#pragma once

#include "layers.cuh"
#include "tc_common.cuh"

namespace uno {

constexpr int ATC_THREADS = 192;
constexpr int ATC_QROWS = 128;
constexpr int ATC_KT = 64;          // keys per tile = one KV page
constexpr int ATC_PAGE_PF = 64;     // page numbers a CTA fetches up front
constexpr int ST_ATTN_TIMEOUT = 16;
constexpr int ATC_PF_LANES = 8;     // producer-warp lanes issuing the L2 prefetch
// Floats per query row of a split partial: O[HD], m, l, padded so that every
// row starts on a 16-byte boundary (rows are written with float4 stores).
__host__ __device__ constexpr int atc_ws_row(int hd) { return hd + 4; }

struct AttnTcParams {
  const f16* q; int ld_q;           // rotated q rows [M, H * HD] (fp16 hi; lo rows q_lo_row below)
  int q_lo_row;
  bf16* out; int ld_out;            // [M, H * HD]
  bf16* out_lo;                     // rounding residual rows (split GEMM input) or null
  int layer, H, Hkv, n_pages, pages_per_req;
  const int32_t* page_table;
  float scale_log2;                 // log2(e) / sqrt(HD)
  int rows_per_req;
  const int32_t* row_pos; const int32_t* row_slot;
  RowKeys keys;                     // per-row key ranges (block-causal rule)
  int n_splits, n_qtiles;
  float* ws;                        // split partials [group][split][128][HD + 4]
  int32_t* status;
  // weights of the projection after the attention, prefetched into L2 by the
  // producer warp's idle lanes while the KV stream leaves HBM bandwidth
  // unused (null: none); 16-byte aligned, a multiple of 16 bytes
  const char* l2_pf; unsigned long long l2_pf_bytes;
};

template <int HD>
struct AtcCfg {
  static constexpr int NB = HD / 64;
  static constexpr int Q_BYTES = ATC_QROWS * HD * 2;
  static constexpr int KV_BYTES = ATC_KT * HD * 2;      // K or V of one stage
  static constexpr int P_BYTES = ATC_QROWS * ATC_KT * 2;
  // stages of K hi, K lo and V beside q hi/lo and one P tile: three for
  // head_dim 128 (224 KB), six for 64
  static constexpr int STAGES = HD <= 64 ? 6 : 3;
  static constexpr int SMEM = 2 * Q_BYTES + STAGES * 3 * KV_BYTES + P_BYTES + 1024 + 256;
  static constexpr int TMEM_COLS = 256;       // 2 score tiles + the output accumulator
  static constexpr int S_COL = 0;             // score tiles at columns 0, 64
  static constexpr int O_COL = 2 * ATC_KT;    // output accumulator at 128 .. 128 + HD
};

// One query row of the output in bf16, plus its rounding residual if `lo`.
template <int HD>
__device__ __forceinline__ void attn_store_row(bf16* dst, bf16* lo, const float* o, float inv) {
#pragma unroll
  for (int d = 0; d < HD; d += 2) {
    const float a = o[d] * inv, b = o[d + 1] * inv;
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    *reinterpret_cast<__nv_bfloat162*>(dst + d) = h;
    if (lo)
      *reinterpret_cast<__nv_bfloat162*>(lo + d) =
          __floats2bfloat162_rn(a - __low2float(h), b - __high2float(h));
  }
}

template <int HD>
__global__ void __launch_bounds__(ATC_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap kvmap, const __grid_constant__ CUtensorMap qmap,
                   const AttnTcParams p) {
  using C = AtcCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* sQ = smem;                                   // q hi: NB boxes [128 rows x 64]
  uint8_t* sQl = sQ + C::Q_BYTES;                       // q lo
  uint8_t* sK = sQl + C::Q_BYTES;                       // [STAGES] K hi: NB boxes [64 keys x 64]
  uint8_t* sKl = sK + C::STAGES * C::KV_BYTES;          // [STAGES] K lo
  uint8_t* sV = sKl + C::STAGES * C::KV_BYTES;          // [STAGES] V
  // one P tile [128 rows x 64 keys]: P(i) is written only after PV(i-1), its
  // previous reader, has completed (the softmax waits for that anyway)
  uint8_t* sP = sV + C::STAGES * C::KV_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + C::P_BYTES);
  uint64_t* kv_full = bars;                             // [STAGES]
  uint64_t* kv_empty = bars + C::STAGES;                // [STAGES]
  uint64_t* s_full = bars + 2 * C::STAGES;              // [2]
  uint64_t* s_empty = s_full + 2;                       // [2] (4 warps)
  uint64_t* p_full = s_empty + 2;                       // [2] (4 warps)
  uint64_t* o_full = p_full + 2;                        // one phase per PV(i)
  uint64_t* drain = o_full + 1;
  uint64_t* q_full = drain + 1;                         // q hi and lo landed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(q_full + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  volatile int* s_ok = reinterpret_cast<volatile int*>(s_tmem + 4);   // [4]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // barriers, TMEM and descriptors depend on no earlier kernel: set up
  // before the wait
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 4);
      mbar_init(&p_full[b], 4);
    }
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    mbar_init(q_full, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(s_tmem)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (warp == 4 && lane == 0) {
    prefetch_map(&kvmap);
    prefetch_map(&qmap);
  }
  if (p.l2_pf && warp == 4 && lane >= 1 && lane <= ATC_PF_LANES) {
    // this CTA's share of the next projection's weights, in 16-byte units
    const unsigned long long units = p.l2_pf_bytes >> 4;
    const unsigned long long ctas = (unsigned long long)gridDim.x * gridDim.y * gridDim.z;
    const unsigned long long cta = blockIdx.x + gridDim.x * (blockIdx.y + (unsigned long long)gridDim.y * blockIdx.z);
    const unsigned long long parts = ctas * ATC_PF_LANES, part = cta * ATC_PF_LANES + (lane - 1);
    const unsigned long long u0 = units * part / parts, u1 = units * (part + 1) / parts;
    if (u1 > u0)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p.l2_pf + (u0 << 4)),
                   "r"((unsigned)((u1 - u0) << 4))
                   : "memory");
  }
  pdl_wait();
  const int split = blockIdx.x, qt = blockIdx.y, z = blockIdx.z;
  const int req = z / p.Hkv, kvh = z % p.Hkv;
  const int G = p.H / p.Hkv;
  const int TQ = ATC_QROWS / G;                  // tokens per query tile
  const int tok0 = qt * TQ;
  const int ntok = min(TQ, p.rows_per_req - tok0);
  const int nq = ntok * G;
  const int row0 = req * p.rows_per_req + tok0;
  // each query row's key ranges (warps 0-3, one row per thread): clean keys
  // [0, qlim), noised keys [qlo2, qhi2)
  int qlim = 0, qlo2 = 0, qhi2 = 0;
  if (warp < 4 && threadIdx.x < nq) p.keys.ranges(p.row_pos, row0 + threadIdx.x / G, qlim, qlo2, qhi2);
  // the tile's key list: pages of the clean range, then of the noised range
  const KeyTiles kt = p.keys.tiles(p.row_pos, p.row_slot, row0, ntok, ATC_KT, p.pages_per_req);
  if (kt.overflow && threadIdx.x == 0 && split == 0) raise_status(p.status, ST_POS_OVERFLOW);
  const int ntiles = kt.n1 + kt.n2;
  const int t_begin = (int)((long long)ntiles * split / p.n_splits);
  const int t_end = (int)((long long)ntiles * (split + 1) / p.n_splits);
  const int n = t_end - t_begin;
  auto page_of_tile = [&](int t) {   // pool page of tile t of the list
    return t < kt.n1 ? p.page_table[(size_t)kt.slot1 * p.pages_per_req + t]
                     : p.page_table[(size_t)kt.slot2 * p.pages_per_req + kt.p2 + (t - kt.n1)];
  };

  // the split's page numbers, fetched in one round while the q rows load
  __shared__ int s_pages[ATC_PAGE_PF];
  if (warp == 4) {
    for (int i = lane; i < min(n, ATC_PAGE_PF); i += 32) s_pages[i] = page_of_tile(t_begin + i);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // q hi and lo tiles: rows (token, head of the group) as a 3-D box of the
      // [rows, H, HD] q buffer; rows past the request are masked, not stored
      if (n > 0) {
        mbar_expect_tx(q_full, 2 * C::Q_BYTES);
#pragma unroll
        for (int b = 0; b < C::NB; ++b) {
          tma_load_3d(sQ + b * (ATC_QROWS * 128), &qmap, q_full, b * 64, kvh * G, row0);
          tma_load_3d(sQl + b * (ATC_QROWS * 128), &qmap, q_full, b * 64, kvh * G, p.q_lo_row + row0);
        }
      }
      const uint64_t pol = l2_evict_first_policy();   // K/V are read once per pass
      int issued = 0;
      for (int i = 0; i < n && !*s_abort; ++i) {
        const int stage = i % C::STAGES;
        const uint32_t phase = (uint32_t)(i / C::STAGES) & 1;
        if (!mbar_wait(&kv_empty[stage], phase ^ 1)) { *s_abort = 1; break; }
        mbar_expect_tx(&kv_full[stage], 3 * C::KV_BYTES);
        const int page = i < ATC_PAGE_PF ? s_pages[i] : page_of_tile(t_begin + i);
        // pool rows of the page's K hi, K lo and V planes for this kv head
        const int rk = (((p.layer * p.n_pages + page) * 3 + 0) * p.Hkv + kvh) * KV_PAGE;
        const int rkl = rk + p.Hkv * KV_PAGE;
        const int rv = rkl + p.Hkv * KV_PAGE;
#pragma unroll
        for (int b = 0; b < C::NB; ++b) {
          const int o = stage * C::KV_BYTES + b * (ATC_KT * 128);
          tma_load_2d_stream(sK + o, &kvmap, &kv_full[stage], b * 64, rk, pol);
          tma_load_2d_stream(sKl + o, &kvmap, &kv_full[stage], b * 64, rkl, pol);
          tma_load_2d_stream(sV + o, &kvmap, &kv_full[stage], b * 64, rv, pol);
        }
        ++issued;
      }
      if (*s_abort) {
        for (int i = max(0, issued - C::STAGES); i < issued; ++i)
          mbar_wait(&kv_full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1);
      }
      if (n > 0) mbar_wait(q_full, 0);   // no copy in flight past this point
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_f16(ATC_QROWS, ATC_KT);
      constexpr uint32_t idesc_pv = idesc_f16(ATC_QROWS, HD) | (1u << 16);   // B MN-major
      bool issued_any = false;
      bool ok = mbar_wait(q_full, 0);
      auto qk = [&](int i) -> bool {
        const int stage = i % C::STAGES, sb = i & 1;
        if (!mbar_wait(&kv_full[stage], (uint32_t)(i / C::STAGES) & 1)) return false;
        if (!mbar_wait(&s_empty[sb], ((uint32_t)(i >> 1) & 1) ^ 1)) return false;
        tc_fence_after();
        const uint32_t d = tmem + C::S_COL + sb * ATC_KT;
        // S = q_hi K_hi^T + q_lo K_hi^T + q_hi K_lo^T (the lo x lo term is below
        // fp32 rounding of S)
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const int b = ks >> 2, kk = ks & 3;
          const int o = stage * C::KV_BYTES + b * (ATC_KT * 128);
          const uint64_t kh = sdesc_k128(smem_u32(sK + o) + kk * 32);
          const uint64_t kl = sdesc_k128(smem_u32(sKl + o) + kk * 32);
          const uint64_t qh = sdesc_k128(smem_u32(sQ + b * (ATC_QROWS * 128)) + kk * 32);
          const uint64_t ql = sdesc_k128(smem_u32(sQl + b * (ATC_QROWS * 128)) + kk * 32);
          mma_f16(d, qh, kh, idesc_qk, ks > 0 ? 1u : 0u);
          mma_f16(d, ql, kh, idesc_qk, 1u);
          mma_f16(d, qh, kl, idesc_qk, 1u);
        }
        issued_any = true;
        mma_commit(&s_full[sb]);
        return true;
      };
      ok = ok && qk(0);
      for (int i = 0; i < n && ok; ++i) {
        if (i + 1 < n && !qk(i + 1)) { ok = false; break; }
        const int stage = i % C::STAGES, b2 = i & 1;
        // P(i) written (and O rescaled, if the softmax warps moved the max)
        if (!mbar_wait(&p_full[b2], (uint32_t)(i >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        // O accumulates in TMEM across tiles
#pragma unroll
        for (int ks = 0; ks < ATC_KT / 16; ++ks)
          mma_f16(tmem + C::O_COL, sdesc_k128(smem_u32(sP) + ks * 32),
                   sdesc_mn128(smem_u32(sV + stage * C::KV_BYTES) + ks * 2048, ATC_KT * 128),
                   idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        mma_commit(o_full);            // phase i completes when PV(i) has
        mma_commit(&kv_empty[stage]);
      }
      if (!ok) {
        *s_abort = 1;
        if (issued_any) {
          mma_commit(drain);
          mbar_wait(drain, 0);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int r = threadIdx.x;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    // Lazy rescaling: P is formed against a reference max m that moves only
    // when a tile's max exceeds it by more than RESCALE_LOG2 (so P <= 2^8);
    // O then stays in TMEM and is rewritten only on those (rare) moves.
    // PV(i) can start only after the softmax signals P(i), so when tile i is
    // in hand at most PV(0..i-1) have completed: waiting for the o_full phase
    // of PV(i-1) by parity is unambiguous.
    constexpr float RESCALE_LOG2 = 8.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int sb = i & 1;
      bool w = !*s_abort && mbar_wait(&s_full[sb], (uint32_t)(i >> 1) & 1);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      float s[ATC_KT];
      tmem_ld32(lane_base + C::S_COL + sb * ATC_KT, s);
      tmem_ld32(lane_base + C::S_COL + sb * ATC_KT + 32, s + 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);
      // raw scores; keys outside the row's range of this tile's segment -> -inf
      // (only the edge tiles of a range need the test)
      const int ti = t_begin + i;
      const bool seg2 = ti >= kt.n1;
      const int kp0 = (seg2 ? kt.p2 + (ti - kt.n1) : ti) * ATC_KT;
      const int klo = seg2 ? qlo2 : 0, khi = seg2 ? qhi2 : qlim;
      float mx = -INFINITY;
      if (kp0 >= klo && kp0 + ATC_KT <= khi) {
#pragma unroll
        for (int j = 0; j < ATC_KT; ++j) mx = fmaxf(mx, s[j]);
      } else {
#pragma unroll
        for (int j = 0; j < ATC_KT; ++j) {
          if (kp0 + j < klo || kp0 + j >= khi) s[j] = -INFINITY;
          mx = fmaxf(mx, s[j]);
        }
      }
      mx *= p.scale_log2;             // log2 units (the scale is positive)
      bool pv_done = false;           // PV(i-1) known complete
      const bool need = mx > m + RESCALE_LOG2;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m;
        if (i > 0) {
          bool w2 = !*s_abort && mbar_wait(o_full, (uint32_t)(i - 1) & 1);
          if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
          pv_done = true;
          tc_fence_after();
          const float corr = (m_new == m) ? 1.f : exp2f(m - m_new);   // m = -inf: O row is 0
#pragma unroll 1
          for (int c0 = 0; c0 < HD; c0 += 32) {
            float v[32];
            tmem_ld32(lane_base + C::O_COL + c0, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= corr;
            tmem_st32(lane_base + C::O_COL + c0, v);
          }
          l *= corr;
        }
        m = m_new;
      }
      // P = 2^(s * scale - m) <= 2^RESCALE_LOG2 by the hardware ex2 (P is
      // rounded to fp16 next, far coarser than its error); a row with no key
      // yet (m = -inf) has s = -inf everywhere and gets P = 0
      const float nm = (m == -INFINITY) ? 0.f : -m;
      float psum = 0.f;
      uint32_t pk[ATC_KT / 2];
#pragma unroll
      for (int j = 0; j < ATC_KT; j += 2) {
        const float a = fast_exp2(fmaf(s[j], p.scale_log2, nm));
        const float b = fast_exp2(fmaf(s[j + 1], p.scale_log2, nm));
        const __half2 h2 = __floats2half2_rn(a, b);
        psum += __low2float(h2) + __high2float(h2);    // the P the MMA will use
        pk[j / 2] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      l += psum;
      // the P tile was last read by PV(i-1): wait for it before overwriting
      if (i > 0 && !pv_done) {
        bool w2 = !*s_abort && mbar_wait(o_full, (uint32_t)(i - 1) & 1);
        if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
      }
      // P row -> shared memory (K-major over keys, 128-byte swizzle)
      uint8_t* prow = sP + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    float o[HD];
#pragma unroll
    for (int d = 0; d < HD; ++d) o[d] = 0.f;
    if (ok && n > 0) {
      bool w2 = !*s_abort && mbar_wait(o_full, (uint32_t)(n - 1) & 1);
      if (__all_sync(0xffffffffu, w2)) {
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) tmem_ld32(lane_base + C::O_COL + c0, o + c0);
        tc_fence_before();
      } else {
        ok = false;
      }
    }
    // epilogue-uniform decision
    if (lane == 0) s_ok[warp] = ok ? 1 : 0;
    epi_bar();
    const bool all_ok = s_ok[0] && s_ok[1] && s_ok[2] && s_ok[3];
    if (!all_ok) {
      *s_abort = 1;
    } else if (p.n_splits == 1) {
      if (r < nq) {
        const int tk = r / G, g = r % G;
        const size_t oo = (size_t)(row0 + tk) * p.ld_out + (size_t)(kvh * G + g) * HD;
        attn_store_row<HD>(p.out + oo, p.out_lo ? p.out_lo + oo : nullptr, o, 1.f / l);
      }
    } else if (r < nq) {
      // split partial (o unnormalised, m in log2 units, l); merged by
      // attn_merge_kernel
      const size_t group = (size_t)z * p.n_qtiles + qt;
      float* w = p.ws + ((group * p.n_splits + split) * ATC_QROWS + r) * atc_ws_row(HD);
#pragma unroll
      for (int d = 0; d < HD; d += 4)
        *reinterpret_cast<float4*>(w + d) = make_float4(o[d], o[d + 1], o[d + 2], o[d + 3]);
      w[HD] = m;
      w[HD + 1] = l;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*s_abort && threadIdx.x == 0) raise_status(p.status, ST_ATTN_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS));
  }
}

// Merge of the split partials: one CTA per (ATC_MERGE_ROWS query rows,
// group), one thread per (row, head_dim element).  Every thread loads all
// splits' (m, l) (the same addresses across a row) together with its own O
// column, so the merge is one round of loads; the splits are added in split
// order.
// Registers stay small enough (rows x head_dim threads) that a GEMM CTA of
// the next projection fits on the same SM and starts its weight stream.
constexpr int ATC_MAX_SPLITS = 24;
constexpr int ATC_MERGE_ROWS = 2;
template <int HD>
__global__ void __launch_bounds__(HD * ATC_MERGE_ROWS) attn_merge_kernel(const AttnTcParams p) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * ATC_MERGE_ROWS + threadIdx.y, group = blockIdx.y;
  const int z = group / p.n_qtiles, qt = group % p.n_qtiles;
  const int req = z / p.Hkv, kvh = z % p.Hkv;
  const int G = p.H / p.Hkv;
  const int TQ = ATC_QROWS / G;
  const int tok0 = qt * TQ;
  const int ntok = min(TQ, p.rows_per_req - tok0);
  if (r < ntok * G) {
    const int d = threadIdx.x;
    const size_t sstride = (size_t)ATC_QROWS * atc_ws_row(HD);
    const float* wg = p.ws + ((size_t)group * p.n_splits * ATC_QROWS + r) * atc_ws_row(HD);
    float ms[ATC_MAX_SPLITS], ls[ATC_MAX_SPLITS], os[ATC_MAX_SPLITS];
#pragma unroll
    for (int s = 0; s < ATC_MAX_SPLITS; ++s) {
      if (s < p.n_splits) {
        const float2 ml = *reinterpret_cast<const float2*>(wg + s * sstride + HD);
        ms[s] = ml.x;
        ls[s] = ml.y;
        os[s] = wg[s * sstride + d];
      } else {
        ms[s] = -INFINITY;
        ls[s] = 0.f;
        os[s] = 0.f;
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < ATC_MAX_SPLITS; ++s) M = fmaxf(M, ms[s]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int s = 0; s < ATC_MAX_SPLITS; ++s) {
      const float w = (ms[s] == -INFINITY) ? 0.f : exp2f(ms[s] - M);
      L += ls[s] * w;
      O += os[s] * w;
    }
    const int row0 = req * p.rows_per_req + tok0;
    const int tk = r / G, g = r % G;
    const size_t oo = (size_t)(row0 + tk) * p.ld_out + (size_t)(kvh * G + g) * HD + d;
    store_split<bf16>(p.out, p.out_lo, oo, O / L);
  }
}

}  // namespace uno
