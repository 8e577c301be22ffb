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
//           tile; O += P V (M=128, N=head_dim, A operand P from TMEM, B
//           operand MN-major) into one TMEM accumulator for the whole key
//           range; the score tile is free again when PV has read its P;
//   warps 0-3 (thread = query row): read the score row, softmax in the log2
//           domain against a reference max that moves (rescaling O in TMEM)
//           only when a tile's max exceeds it by more than 2^8, and write P
//           (fp16) into TMEM over the scores just read, so the softmax of one
//           tile runs while the PV of the one before it does.
// With several key splits each CTA writes (m, l, O) partials and
// attn_merge_kernel (ATC_MERGE_ROWS query rows per CTA) adds them in split
// order.  Every wait is bounded.  While it runs, idle lanes of the producer
// warp prefetch part of the next projection's weights into L2.
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
  // completion counter of the kernel that wrote q and the new K/V rows (null:
  // pdl_wait instead) and its CTA count; for the merge kernel, the
  // attention's counter
  const unsigned* dep; unsigned dep_count;
  unsigned long long dep_limit_ns;
  unsigned* done;                   // counter every CTA adds to at its end (or null)
};

// The inputs' dependency: one thread polls the counter (the TMA producer
// lane, which then orders its later bulk copies after the generic stores it
// observed) and the CTA meets it at a barrier; or the grid dependency.
__device__ __forceinline__ void attn_dep_wait(const AttnTcParams& p, bool poller) {
  if (p.dep) {
    if (poller) {
      if (!dep_wait(p.dep, p.dep_count, p.dep_limit_ns)) raise_status(p.status, ST_DEP_TIMEOUT);
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncthreads();
  } else {
    pdl_wait();
  }
}

template <int HD>
struct AtcCfg {
  static constexpr int NB = HD / 64;
  static constexpr int Q_BYTES = ATC_QROWS * HD * 2;
  static constexpr int KV_BYTES = ATC_KT * HD * 2;      // K or V of one stage
  // stages of K hi, K lo and V beside q hi/lo (P lives in tensor memory):
  // three for head_dim 128 (209 KB), six for 64 (177 KB), so that a CTA fits
  // on an SM beside a q|k|v epilogue CTA and starts while that epilogue runs
  static constexpr int STAGES = HD <= 64 ? 6 : 3;
  static constexpr int SMEM = 2 * Q_BYTES + STAGES * 3 * KV_BYTES + 1024 + 256;
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

// At most 128 registers a thread: two of its warps and two q|k|v epilogue
// warps (128 each) then fill one SM sub-partition's 16,384 registers, so
// the CTA starts beside an epilogue CTA.
template <int HD>
__global__ void __maxnreg__(128)
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + C::STAGES * C::KV_BYTES);
  uint64_t* kv_full = bars;                             // [STAGES]
  uint64_t* kv_empty = bars + C::STAGES;                // [STAGES]
  uint64_t* s_full = bars + 2 * C::STAGES;              // [2]
  uint64_t* s_empty = s_full + 2;                       // [2] (PV of the tile held there)
  uint64_t* p_full = s_empty + 2;                       // [2] (4 warps)
  uint64_t* o_full = p_full + 2;                        // [2] one phase per PV of a tile there
  uint64_t* drain = o_full + 2;
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
      mbar_init(&s_empty[b], 1);
      mbar_init(&p_full[b], 4);
    }
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
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
  // With a completion counter (the fused pass) the row tables and the page
  // table are complete when this kernel starts: the pass's first kernel after
  // build_rows lets the next one launch only once build_rows has completed.
  // The key list and its pages are then set up, and the split's first page,
  // if no row of this pass writes it, starts loading while the q|k|v
  // epilogue still runs (the table loads go through L2: before the
  // dependency wait L1 may still hold an earlier pass's lines).  Without a
  // counter everything follows the grid dependency.
  const bool early = p.dep != nullptr;
  if (!early) pdl_wait();
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
    return t < kt.n1 ? __ldcg(p.page_table + (size_t)kt.slot1 * p.pages_per_req + t)
                     : __ldcg(p.page_table + (size_t)kt.slot2 * p.pages_per_req + kt.p2 + (t - kt.n1));
  };

  // the split's page numbers, fetched in one round while the q rows load
  __shared__ int s_pages[ATC_PAGE_PF];
  int n_safe = 0;   // leading tiles of the split loadable before the wait (warp 4)
  if (warp == 4) {
    for (int i = lane; i < min(n, ATC_PAGE_PF); i += 32) s_pages[i] = page_of_tile(t_begin + i);
    if (early && !p.keys.cslot && !p.keys.blk) {
      // every key is in the request's slot and this pass writes K/V only at
      // its rows' positions there: whole pages below the lowest of those
      // positions hold cached keys alone
      int lowest = 0x7fffffff;
      for (int k = lane; k < p.rows_per_req; k += 32) {
        const int ps = __ldcg(p.row_pos + req * p.rows_per_req + k);
        if (ps >= 0) lowest = min(lowest, ps);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lowest = min(lowest, __shfl_xor_sync(0xffffffffu, lowest, o));
      // one page: loading more of them early slowed the epilogue beside it
      n_safe = max(0, min(min(n, 1), lowest / ATC_KT - t_begin));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // K hi, K lo and V of list entry i into its ring stage (producer lane)
  auto issue_tile = [&](int i, uint64_t pol) -> bool {
    const int stage = i % C::STAGES;
    const uint32_t phase = (uint32_t)(i / C::STAGES) & 1;
    if (!mbar_wait(&kv_empty[stage], phase ^ 1)) return false;
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
    return true;
  };
  int issued = 0;                 // tiles issued (producer lane)
  uint64_t pol = 0;               // K/V are read once per pass: evict first
  if (warp == 4 && lane == 0) {
    pol = l2_evict_first_policy();
    while (issued < n_safe && issue_tile(issued, pol)) ++issued;
  }
  if (early) attn_dep_wait(p, warp == 4 && lane == 0);

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
      if (issued < n_safe) *s_abort = 1;   // an early stage wait gave up
      for (int i = issued; i < n && !*s_abort; ++i) {
        if (!issue_tile(i, pol)) { *s_abort = 1; break; }
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
        // O accumulates in TMEM across tiles; P(i) (fp16, 16 keys per 8
        // columns) sits over the first half of its score tile
#pragma unroll
        for (int ks = 0; ks < ATC_KT / 16; ++ks)
          mma_f16_ts(tmem + C::O_COL, tmem + C::S_COL + b2 * ATC_KT + ks * 8,
                     sdesc_mn128(smem_u32(sV + stage * C::KV_BYTES) + ks * 2048, ATC_KT * 128),
                     idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&o_full[b2]);       // completes when PV(i) (and every MMA before it) has
        mma_commit(&kv_empty[stage]);
        mma_commit(&s_empty[b2]);      // P(i) read: the score tile is free
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
    // PV(i) can start only after the softmax signals P(i), and the softmax may
    // run ahead of the PVs, so their completions are counted per score
    // buffer: tile j's PV is completion j / 2 of o_full[j % 2], and a PV of
    // the same buffer two tiles on cannot complete before the softmax has
    // moved past tile j + 1, so a wait by parity is unambiguous.
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
      const bool need = mx > m + RESCALE_LOG2;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m;
        if (i > 0) {
          bool w2 = !*s_abort && mbar_wait(&o_full[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1);
          if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
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
      // P row -> tensor memory over the scores just read (this thread's lane;
      // the tile is not rewritten before PV(i) has read it)
      tmem_st32u(lane_base + C::S_COL + sb * ATC_KT, pk);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    if (ok && n > 0) {
      bool w2 = !*s_abort && mbar_wait(&o_full[(n - 1) & 1], (uint32_t)((n - 1) >> 1) & 1);
      if (!__all_sync(0xffffffffu, w2)) ok = false;
    }
    // epilogue-uniform decision
    if (lane == 0) s_ok[warp] = ok ? 1 : 0;
    epi_bar();
    const bool all_ok = s_ok[0] && s_ok[1] && s_ok[2] && s_ok[3];
    if (!all_ok) {
      *s_abort = 1;
    } else {
      // O (rows past the tile's queries read too: the TMEM load is warp-wide)
      // 32 columns at a time, so that few registers hold it
      tc_fence_after();
      const int tk = r / G, g = r % G;
      const size_t oo = (size_t)(row0 + tk) * p.ld_out + (size_t)(kvh * G + g) * HD;
      const size_t group = (size_t)z * p.n_qtiles + qt;
      float* w = p.ws + ((group * p.n_splits + split) * ATC_QROWS + r) * atc_ws_row(HD);
      const float inv = 1.f / l;
#pragma unroll 1
      for (int c0 = 0; c0 < HD; c0 += 32) {
        float o[32];
        if (n > 0) {
          tmem_ld32(lane_base + C::O_COL + c0, o);
        } else {
#pragma unroll
          for (int d = 0; d < 32; ++d) o[d] = 0.f;
        }
        if (r >= nq) continue;
        if (p.n_splits == 1) {
          attn_store_row<32>(p.out + oo + c0, p.out_lo ? p.out_lo + oo + c0 : nullptr, o, inv);
        } else {
          // split partial (o unnormalised, m in log2 units, l); merged by
          // attn_merge_kernel
#pragma unroll
          for (int d = 0; d < 32; d += 4)
            *reinterpret_cast<float4*>(w + c0 + d) = make_float4(o[d], o[d + 1], o[d + 2], o[d + 3]);
        }
      }
      tc_fence_before();
      if (p.n_splits > 1 && r < nq) {
        w[HD] = m;
        w[HD + 1] = l;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*s_abort && threadIdx.x == 0) raise_status(p.status, ST_ATTN_TIMEOUT);
  dep_signal_synced(p.done);        // the split partials are stored
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
  attn_dep_wait(p, threadIdx.x == 0 && threadIdx.y == 0);
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
        // through L2: with a completion counter there is no grid wait to
        // drop L1 lines of an earlier pass
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(wg + s * sstride + HD));
        ms[s] = ml.x;
        ls[s] = ml.y;
        os[s] = __ldcg(wg + s * sstride + d);
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
