// gated_lora_linear for many token rows (the max-batch and prefill passes):
// tokens in the MMA's M, weights in its N.
//
// With hi/lo split inputs (x = hi + lo, see gemm_tc.cuh) and the weights as
// the M operand, the MMA's N holds 128 token rows twice, so a stage carries
// 32 KB of weights and 64 KB of tokens per 128 x 256 x 128 product.  Here the
// token tile is the M operand (128 rows) and the weight tile the N operand
// (256 rows): the hi and lo token tiles are two MMAs into one accumulator, so
// each weight k-block serves both, and a stage of one 64-wide k-block holds
// 16 + 16 KB of tokens and 32 KB of weights for the same flops as the 96 KB
// of the other form: a third less traffic from L2 for a pass that is
// tensor-bound.  Not DUMP mode; the schedule (stream-K, m-tile groups), the
// barriers, the bounded waits and the in-kernel fixup are those of
// gemm_tc_kernel with rows and columns exchanged.
#pragma once

#include "gemm_tc.cuh"

namespace uno {

constexpr int TK_BN = 256;           // weight rows per tile (MMA N)
constexpr int TK_BM = 128;           // token rows per tile (MMA M)
struct TkCfg {
  static constexpr int A_SUB = TK_BM * TC_BK * 2;          // 16 KB: one token tile (hi or lo)
  static constexpr int B_BYTES = TK_BN * TC_BK * 2;        // 32 KB: the weight tile
  static constexpr int STAGE_BYTES = 2 * A_SUB + B_BYTES;  // 64 KB
  static constexpr int STAGES = 3;
  static constexpr int TMEM_COLS = 2 * TK_BN;              // two accumulators: all 512 columns
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

// 16 consecutive fp32 output columns n .. n + 15 of token row m (row and
// columns in range; the host checks 16-byte alignment of every row): stored
// scaled by alpha, or added to what is there (the residual stream).
__device__ __forceinline__ void tk_store16(const TcParams& p, int m, int n, const float (&v)[16]) {
  float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (size_t)m * p.ldo + n);
  float4 w[4];
  if (p.epi == EPI_ADD_F32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = __ldcg(dst + q);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      w[q].x += v[4 * q]; w[q].y += v[4 * q + 1]; w[q].z += v[4 * q + 2]; w[q].w += v[4 * q + 3];
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = make_float4(v[4 * q] * p.alpha, v[4 * q + 1] * p.alpha, v[4 * q + 2] * p.alpha,
                         v[4 * q + 3] * p.alpha);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = w[q];
}
// The same for columns that may run past N (scalar, per element).
__device__ __forceinline__ void tk_store16_edge(const TcParams& p, int m, int n, const float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (n + i < p.N) tc_store(p, m, n + i, v[i]);
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    gemm_tokm_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  using C = TkCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  // stage s: [token hi 16 KB][token lo 16 KB][weights 32 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                      // [STAGES] TMA -> MMA
  uint64_t* empty = bars + C::STAGES;         // [STAGES] MMA -> TMA
  uint64_t* tfull = bars + 2 * C::STAGES;     // [2] MMA -> epilogue
  uint64_t* tempty = tfull + 2;               // [2] epilogue -> MMA
  uint64_t* drain = tempty + 2;               // MMA drain on abort
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(s_tmem + 2);
  volatile int* s_ok = reinterpret_cast<volatile int*>(s_tmem + 4);   // [2][4]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KBt = p.KB + p.RB;
  // schedule: as gemm_tc_kernel's (m-tile groups when mgroups > 0)
  const bool grp = p.mgroups > 0;
  const int mt_fix = grp ? (int)blockIdx.x % p.m_tiles : 0;
  const int me = grp ? (int)blockIdx.x / p.m_tiles : (int)blockIdx.x;
  const int nsplit = grp ? p.mgroups : p.grid;
  const int vunits = grp ? p.n_tiles * KBt : p.units;
  const int u0 = sk_start(me, vunits, nsplit);
  const int u1 = sk_start(me + 1, vunits, nsplit);
  auto tile_of = [&](int u) { return grp ? (u / KBt) * p.m_tiles + mt_fix : u / KBt; };
  auto seg_of = [&](int n_row) {
    int sg = 0;
    for (int s = 1; s < p.nseg; ++s)
      if (n_row >= p.seg[s].n0) sg = s;
    return sg;
  };
  uint64_t pol_stream = 0;   // set by the TMA issuer
  // the weight tile of unit u: two 128-row boxes of W (or of LoRA-B)
  auto load_w = [&](int u, int stage) {
    const int t = tile_of(u), kb = u % KBt;
    const int n_row = (t / p.m_tiles) * TK_BN;
    const int sg = seg_of(n_row);
    const CUtensorMap* map = kb < p.KB ? &maps.w[sg] : &maps.b[sg];
    const int x = (kb < p.KB ? kb : kb - p.KB) * TC_BK;
    const int y = n_row - p.seg[sg].n0;
    uint8_t* dst = smem + stage * C::STAGE_BYTES + 2 * C::A_SUB;
    tma_load_2d_stream(dst, map, &full[stage], x, y, pol_stream);
    tma_load_2d_stream(dst + TC_A_BYTES, map, &full[stage], x, y + TC_BM, pol_stream);
  };
  // the token tiles of unit u: X (or U), hi rows then lo rows
  auto load_x = [&](int u, int stage) {
    const int t = tile_of(u), kb = u % KBt;
    const int mt = t % p.m_tiles;
    uint8_t* dst = smem + stage * C::STAGE_BYTES;
    if (kb < p.KB) {
      const int x = kb * TC_BK;
      tma_load_2d(dst, &maps.x, &full[stage], x, mt * TK_BM);
      tma_load_2d(dst + C::A_SUB, &maps.x, &full[stage], x, p.lo_off + mt * TK_BM);
    } else {
      const int sg = seg_of((t / p.m_tiles) * TK_BN);
      const int x = p.seg[sg].u_off + (kb - p.KB) * TC_BK;
      tma_load_2d(dst, &maps.u, &full[stage], x, mt * TK_BM);
      tma_load_2d(dst + C::A_SUB, &maps.u, &full[stage], x, p.lo_off + mt * TK_BM);
    }
  };
  const int total = u1 - u0;
  const int npre = min(total, C::STAGES);

  if (warp == 4 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);   // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_map(&maps.x);
    for (int s = 0; s < p.nseg; ++s) prefetch_map(&maps.w[s]);
    pol_stream = l2_evict_first_policy();
    // the weights depend on no earlier kernel: their first stages before the wait
    for (int i = 0; i < npre; ++i) {
      mbar_expect_tx(&full[i], C::STAGE_BYTES);
      load_w(u0 + i, i);
    }
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(s_tmem)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  pdl_trigger();
  if (!(warp == 4 && lane == 0)) pdl_wait();

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      pdl_wait();
      for (int i = 0; i < npre; ++i) load_x(u0 + i, i);
      int issued = npre;
      for (int i = npre; i < total && !*s_abort; ++i) {
        const int stage = i % C::STAGES;
        if (!mbar_wait(&empty[stage], ((uint32_t)(i / C::STAGES) & 1) ^ 1)) { *s_abort = 1; break; }
        mbar_expect_tx(&full[stage], C::STAGE_BYTES);
        load_w(u0 + i, stage);
        load_x(u0 + i, stage);
        ++issued;
      }
      if (*s_abort) {
        for (int i = max(0, issued - C::STAGES); i < issued; ++i)
          mbar_wait(&full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(TK_BM, TK_BN);
      int stage = 0, part = 0, issued = 0;
      uint32_t phase = 0;
      for (int u = u0; u < u1 && !*s_abort; ++part) {
        const int kb0 = u % KBt;
        const int kb1 = min(KBt, kb0 + (u1 - u));
        const int buf = part & 1;
        const uint32_t use = (uint32_t)(part >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1) ^ 1)) { *s_abort = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * TK_BN);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + 2 * C::A_SUB;
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            const uint64_t bdesc = sdesc_k128(sb + k * 32);
            mma_f16(d, sdesc_k128(sa + k * 32), bdesc, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            mma_f16(d, sdesc_k128(sa + C::A_SUB + k * 32), bdesc, idesc, 1u);
          }
          ++issued;
          mma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) { *s_abort = 1; break; }
        mma_commit(&tfull[buf]);
        u += kb1 - kb0;
      }
      if (*s_abort && issued) {
        mma_commit(drain);          // tracks every MMA this thread issued
        mbar_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    const int r_local = warp * 32 + lane;     // the thread's token row in the tile
    int part = 0;
    for (int u = u0; u < u1; ++part) {
      const int t = tile_of(u), kb0 = u % KBt;
      const int kb1 = min(KBt, kb0 + (u1 - u));
      u += kb1 - kb0;
      const int buf = part & 1;
      const uint32_t use = (uint32_t)(part >> 1);
      bool ok = !*s_abort && mbar_wait(&tfull[buf], use & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) s_ok[(part & 1) * 4 + warp] = ok ? 1 : 0;
      epi_bar();
      const int pb = (part & 1) * 4;
      if (!(s_ok[pb] && s_ok[pb + 1] && s_ok[pb + 2] && s_ok[pb + 3])) { *s_abort = 1; break; }
      tc_fence_after();
      const int nt = t / p.m_tiles, mt = t % p.m_tiles;
      const int m = mt * TK_BM + r_local;
      const int n0 = nt * TK_BN;
      const bool row_ok = m < p.M;
      const bool whole = kb0 == 0 && kb1 == KBt;
      const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(buf * TK_BN);
      float* wsl = tc_slot(p.ws, blockIdx.x, part == 0 ? 0 : 1, TK_BN);
#pragma unroll 1
      for (int c0 = 0; c0 < TK_BN; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + c0, v);
        if (whole) {
          if (row_ok && n0 + c0 < p.N) {
            if (n0 + c0 + 16 <= p.N) tk_store16(p, m, n0 + c0, v);
            else tk_store16_edge(p, m, n0 + c0, v);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(wsl + (size_t)r_local * TK_BN + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (!whole) {
        __threadfence();
        epi_bar();
        const int vt0 = grp ? (t / p.m_tiles) * KBt : t * KBt;   // the tile's first virtual unit
        const int first = sk_owner(vt0, vunits, nsplit);
        const int last = sk_owner(vt0 + KBt - 1, vunits, nsplit);
        if (threadIdx.x == 0) {
          const unsigned done = atomicAdd(&p.counters[t], 1u);
          const bool is_last = (done == (unsigned)(last - first));
          *s_last = is_last ? 1 : 0;
          if (is_last) p.counters[t] = 0u;
        }
        epi_bar();
        if (*s_last) {
          __threadfence();
          // 16 columns x up to 4 contributors of loads per round, added in
          // CTA order (deterministic)
#pragma unroll 1
          for (int c0 = 0; c0 < TK_BN; c0 += 16) {
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.f;
#pragma unroll 1
            for (int i0 = first; i0 <= last; i0 += 4) {
              float4 w[4][4];
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int i = i0 + c;
                const float4* src = nullptr;
                if (i <= last) {
                  const int slot = (sk_start(i, vunits, nsplit) >= vt0) ? 0 : 1;
                  const int cta = grp ? i * p.m_tiles + mt_fix : i;
                  src = reinterpret_cast<const float4*>(tc_slot(p.ws, cta, slot, TK_BN) +
                                                        (size_t)r_local * TK_BN + c0);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  w[c][q] = src ? __ldcg(src + q) : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
              for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  acc[4 * q] += w[c][q].x; acc[4 * q + 1] += w[c][q].y;
                  acc[4 * q + 2] += w[c][q].z; acc[4 * q + 3] += w[c][q].w;
                }
            }
            if (row_ok && n0 + c0 < p.N) {
              if (n0 + c0 + 16 <= p.N) tk_store16(p, m, n0 + c0, acc);
              else tk_store16_edge(p, m, n0 + c0, acc);
            }
          }
        }
        epi_bar();   // s_last is reused by the next cut part
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*s_abort && threadIdx.x == 0) raise_status(p.status, ST_GEMM_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS));
  }
}

}  // namespace uno
