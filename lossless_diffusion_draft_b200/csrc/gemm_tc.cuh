// Gated-LoRA linear layer on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), for bf16 models.
//
//   Y[m, n] = sum_k X[m, k] W[n, k] + sum_j U[m, uoff + j] Bl[n, j]
//
// Decode passes have few rows (17 per request in the draft pass) and stream
// the whole weight set once per pass, so the kernel is built around the
// weight stream:
//  * swap-AB: a 128-row tile of W is the MMA's A operand (M = 128) and the
//    token rows are its N dimension (NT = 16..256), so no MMA row is wasted
//    on padding tokens;
//  * the LoRA-B product is folded in as extra K-blocks: after the K/64 blocks
//    of (W, X) the same accumulator takes r/64 blocks of (Bl, U), so the
//    base weights and the adapter share one pass over the output tile;
//  * stream-K: the (tile, k-block) units are split evenly over one persistent
//    CTA per SM, so every SM streams the same number of weight bytes whatever
//    the tile count.  Two ways to finish a tile:
//      - in-kernel: a tile cut between CTAs is finished by whichever
//        contributor arrives last (atomic counter, no waiting), which adds
//        the fp32 partials in a fixed order (deterministic) and runs the
//        epilogue;
//      - DUMP: every part goes to its own fp32 slot, tile + cta (unique: both
//        grow together along the unit order), and the CTA moves on; a
//        following epilogue kernel adds a tile's parts in CTA order and fuses
//        whatever comes next.  The reducing CTA's chain of dependent L2
//        round trips then leaves the GEMM's critical path;
//  * warp roles: warp 4 issues TMA loads into a STAGES-deep ring, warp 5
//    issues tcgen05.mma into a double-buffered TMEM accumulator, warps 0-3
//    drain TMEM (tcgen05.ld) and write the epilogue while the next part's
//    MMAs run.
// Every mbarrier wait is bounded (about two seconds of global time); on
// timeout the kernel raises a status bit, stops, waits (bounded) for its own
// TMA copies, frees its TMEM and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "tc_common.cuh"

namespace uno {

constexpr int TC_THREADS = 192;
constexpr int TC_BM = 128;         // weight rows per tile (MMA M)
constexpr int TC_BK = 64;          // k elements per block (128 bytes of bf16)
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;
constexpr int ST_GEMM_TIMEOUT = 8;

constexpr int TC_MAX_SEG = GEMM_MAX_SEG;
struct TcMaps {
  CUtensorMap x;               // activations [rows, K], box {64, NT}
  CUtensorMap u;               // LoRA intermediate [rows, 3r], box {64, NT}
  CUtensorMap w[TC_MAX_SEG];   // weights of each segment [n, K], box {64, 128}
  CUtensorMap b[3];            // LoRA-B of each segment [n, r], box {64, 128}
};

struct TcSeg { int n0, n, u_off; };

struct TcParams {
  int M, N, KB, RB;          // rows, columns, units (KPS k-blocks) of K and of r (0: no LoRA)
  int n_tiles, m_tiles;
  int nseg; TcSeg seg[TC_MAX_SEG];
  int units, grid;           // stream-K: units = tiles * (KB + RB), split over grid CTAs
  // m-tile groups (0: none).  With several token m-tiles, grid = mgroups *
  // m_tiles: CTA b takes m-tile b % m_tiles, and the mgroups groups split the
  // units of one m-tile's row of tiles (n_tiles * (KB + RB)) stream-K style,
  // so the CTAs of a group read the same weight k-blocks at about the same
  // time (one from HBM, the rest from L2) instead of every CTA re-reading its
  // own weight tile once per m-tile.  Not in DUMP mode.
  int mgroups;
  int max_parts;             // partial slots per tile
  int epi; void* out; int ldo; float alpha; const float* row_gate;
  float* ws; unsigned* counters;   // DUMP: ws holds the part slots [tiles + grid][NT][128]
  int32_t* status;
  int lo_off;                // split mode: row offset of the lo rows of X and U
  void* out_lo;              // EPI_GATED in split mode: lo part of the output (out + lo_off rows)
  // completion counter of the kernel that wrote X (null: pdl_wait instead);
  // DUMP mode only, where X is the one input an earlier kernel wrote
  const unsigned* dep; unsigned dep_count;
  unsigned long long dep_limit_ns;   // give up the counter wait after this long
  const int64_t* out_row;            // EPI_STORE_F32: element offset of each output row (null: m * ldo)
  // DUMP mode: completion counter every CTA adds to once its parts are
  // stored (the epilogue kernel after it waits on it), or null
  unsigned* done;
};

// ---------------------------------------------------------------------------
// Stream-K partition.
// ---------------------------------------------------------------------------
// 32-bit arithmetic: units * grid stays below 2^32 for every launch (the
// host checks), and a 64-bit division is a long software sequence.  Host-
// callable too, so that the partition is checked on the CPU.
__host__ __device__ __forceinline__ int sk_start(int i, int units, int grid) {
  return (int)(((unsigned)i * (unsigned)units) / (unsigned)grid);
}
__host__ __device__ __forceinline__ int sk_owner(int u, int units, int grid) {
  int i = (int)(((unsigned)u * (unsigned)grid) / (unsigned)units);
  while (i + 1 < grid && sk_start(i + 1, units, grid) <= u) ++i;
  while (i > 0 && sk_start(i, units, grid) > u) --i;
  return i;
}

// SPLIT: every activation row x is fed as two bf16 rows hi = bf16(x) and
// lo = bf16(x - hi) (rows lo_off apart in the buffer); the MMA's N covers
// both (2 NT columns) and the epilogue adds column m and column NT + m, so
// the product sees x to ~16 mantissa bits while the weights stream once.
// KPS: 64-element k-blocks per pipeline stage (a unit of stream-K work).  Two
// put 256 contiguous bytes of every weight row in flight together.
template <int NT, bool SPLIT, int KPS>
struct TcCfg {
  static constexpr int NMMA = SPLIT ? 2 * NT : NT;           // MMA N
  static constexpr int B_SUB = NMMA * TC_BK * 2;             // one k-block of activations
  static constexpr int A_BYTES = KPS * TC_A_BYTES;
  static constexpr int B_BYTES = KPS * B_SUB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int MAX_STAGES = 8 / KPS;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > MAX_STAGES ? MAX_STAGES
                                                                         : (200 * 1024) / STAGE_BYTES;
  static constexpr int TMEM_COLS = NMMA < 32 ? 64 : 2 * NMMA;  // two accumulators, power of two
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

// Partial-tile slot of a contributor: its first part uses slot 0, its last
// part slot 1 (parts in between cover whole tiles and need none).
__device__ __forceinline__ float* tc_slot(float* ws, int cta, int slot, int NT) {
  return ws + ((size_t)cta * 2 + slot) * NT * TC_BM;
}

__device__ __forceinline__ void tc_store(const TcParams& p, int m, int n, float v) {
  const size_t o = (size_t)m * p.ldo + n;
  switch (p.epi) {
    case EPI_STORE: reinterpret_cast<bf16*>(p.out)[o] = from_f<bf16>(v * p.alpha); break;
    case EPI_STORE_F32:
      reinterpret_cast<float*>(p.out)[p.out_row ? (size_t)p.out_row[m] + n : o] = v * p.alpha;
      break;
    case EPI_ADD_F32: reinterpret_cast<float*>(p.out)[o] += v; break;
    default: {
      const float y = v * p.alpha * p.row_gate[m];
      const bf16 hi = from_f<bf16>(y);
      reinterpret_cast<bf16*>(p.out)[o] = hi;
      if (p.out_lo) reinterpret_cast<bf16*>(p.out_lo)[o] = from_f<bf16>(y - to_f(hi));
      break;
    }
  }
}

// Rows m0 .. m0 + R - 1 of column n (rows past mrows or a column past N are
// skipped).  The residual-add epilogue reads all R old values before it
// writes any: the compiler cannot tell the rows' addresses apart, and would
// otherwise serialise R load / store round trips.
template <int R>
__device__ __forceinline__ void tc_store_rows(const TcParams& p, int m0, int mrows, int n,
                                              const float (&v)[R]) {
  if (n >= p.N) return;
  if (p.epi == EPI_ADD_F32) {
    float* out = reinterpret_cast<float*>(p.out);
    float old[R];
#pragma unroll
    for (int i = 0; i < R; ++i)
      old[i] = i < mrows ? __ldcg(out + (size_t)(m0 + i) * p.ldo + n) : 0.f;
#pragma unroll
    for (int i = 0; i < R; ++i)
      if (i < mrows) out[(size_t)(m0 + i) * p.ldo + n] = old[i] + v[i];
    return;
  }
#pragma unroll
  for (int i = 0; i < R; ++i)
    if (i < mrows) tc_store(p, m0 + i, n, v[i]);
}

template <int NT, bool SPLIT, bool DUMP, int KPS>
__global__ void __launch_bounds__(TC_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  using C = TcCfg<NT, SPLIT, KPS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
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
  // the split this CTA belongs to (units are virtual with m-tile groups: the
  // k-blocks of one row of tiles, this CTA's m-tile fixed)
  const bool grp = !DUMP && p.mgroups > 0;
  const int mt_fix = grp ? (int)blockIdx.x % p.m_tiles : 0;
  const int me = grp ? (int)blockIdx.x / p.m_tiles : (int)blockIdx.x;
  const int nsplit = grp ? p.mgroups : p.grid;
  const int vunits = grp ? p.n_tiles * KBt : p.units;
  const int u0 = sk_start(me, vunits, nsplit);
  const int u1 = sk_start(me + 1, vunits, nsplit);
  auto tile_of = [&](int u) { return grp ? (u / KBt) * p.m_tiles + mt_fix : u / KBt; };

  // unit u is k-block u % KBt of tile u / KBt; issue i = u - u0 uses
  // ring stage i % STAGES
  auto seg_of = [&](int n_row) {
    int sg = 0;
    for (int s = 1; s < p.nseg; ++s)
      if (n_row >= p.seg[s].n0) sg = s;
    return sg;
  };
  // weight tile of unit u: W, then LoRA-B
  auto coords_a = [&](int u, const CUtensorMap*& map, int& x, int& y) {
    const int t = tile_of(u), kb = u % KBt;
    const int n_row = (t / p.m_tiles) * TC_BM;
    const int sg = seg_of(n_row);
    map = kb < p.KB ? &maps.w[sg] : &maps.b[sg];
    x = (kb < p.KB ? kb : kb - p.KB) * TC_BK * KPS;
    y = n_row - p.seg[sg].n0;
  };
  uint64_t pol_stream = 0;   // set by the TMA issuer
  auto load_a = [&](int u, int stage) {
    const CUtensorMap* map;
    int x, y;
    coords_a(u, map, x, y);
#pragma unroll
    for (int j = 0; j < KPS; ++j)
      tma_load_2d_stream(sA + stage * C::A_BYTES + j * TC_A_BYTES, map, &full[stage], x + j * TC_BK,
                         y, pol_stream);
  };


  auto load_b = [&](int u, int stage) {     // activations: X, then U (hi, lo)
    const int t = tile_of(u), kb = u % KBt;
    const int mt = t % p.m_tiles;
#pragma unroll
    for (int j = 0; j < KPS; ++j) {
      uint8_t* dst = sB + stage * C::B_BYTES + j * C::B_SUB;
      if (kb < p.KB) {
        const int x = (kb * KPS + j) * TC_BK;
        tma_load_2d(dst, &maps.x, &full[stage], x, mt * NT);
        if (SPLIT) tma_load_2d(dst + NT * 128, &maps.x, &full[stage], x, p.lo_off + mt * NT);
      } else {
        const int sg = seg_of((t / p.m_tiles) * TC_BM);
        const int x = p.seg[sg].u_off + ((kb - p.KB) * KPS + j) * TC_BK;
        tma_load_2d(dst, &maps.u, &full[stage], x, mt * NT);
        if (SPLIT) tma_load_2d(dst + NT * 128, &maps.u, &full[stage], x, p.lo_off + mt * NT);
      }
    }
  };
  const int total = u1 - u0;
  const int npre = min(total, C::STAGES);

  // The TMA issuer sets up the barriers and starts the weight stream (the
  // weights depend on no earlier kernel) while warp 0 allocates TMEM: the
  // first stages' copies are under way before the CTA's first barrier.
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
    if (p.dep) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.dep));
    pol_stream = l2_evict_first_policy();
    for (int i = 0; i < npre; ++i) {
      mbar_expect_tx(&full[i], C::STAGE_BYTES);
      load_a(u0 + i, i);
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
  // every thread but the TMA issuer waits for the previous kernel here (the
  // issuer has started the weight stream above).  With a completion
  // counter only the issuer waits, for the X rows: the other threads read
  // nothing an earlier kernel wrote (in DUMP mode they only store parts, and
  // those stores follow MMAs on X tiles loaded after the wait).
  if (!p.dep && !(warp == 4 && lane == 0)) pdl_wait();

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      if (p.dep) {
        if (!dep_wait(p.dep, p.dep_count, p.dep_limit_ns)) raise_status(p.status, ST_DEP_TIMEOUT);
        // the X rows were written by generic stores; the loads below are TMA
        asm volatile("fence.proxy.async.global;" ::: "memory");
      } else {
        pdl_wait();
      }
      for (int i = 0; i < npre; ++i) load_b(u0 + i, i);
      int issued = npre;
      for (int i = npre; i < total && !*s_abort; ++i) {
        const int stage = i % C::STAGES;
        if (!mbar_wait(&empty[stage], ((uint32_t)(i / C::STAGES) & 1) ^ 1)) { *s_abort = 1; break; }
        mbar_expect_tx(&full[stage], C::STAGE_BYTES);
        load_a(u0 + i, stage);
        load_b(u0 + i, stage);
        ++issued;
      }
      if (*s_abort) {
        // wait (bounded) for the copies still in flight: the last
        // min(issued, STAGES) issues
        for (int i = max(0, issued - C::STAGES); i < issued; ++i)
          mbar_wait(&full[i % C::STAGES], (uint32_t)(i / C::STAGES) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(TC_BM, C::NMMA);
      int stage = 0, part = 0, issued = 0;
      uint32_t phase = 0;
      for (int u = u0; u < u1 && !*s_abort; ++part) {
        const int kb0 = u % KBt;
        const int kb1 = min(KBt, kb0 + (u1 - u));
        const int buf = part & 1;
        const uint32_t use = (uint32_t)(part >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1) ^ 1)) { *s_abort = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * C::NMMA);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < KPS; ++j) {
            const uint32_t a = smem_u32(sA + stage * C::A_BYTES + j * TC_A_BYTES);
            const uint32_t b = smem_u32(sB + stage * C::B_BYTES + j * C::B_SUB);
#pragma unroll
            for (int k = 0; k < TC_BK / 16; ++k)
              mma_f16(d, sdesc_k128(a + k * 32), sdesc_k128(b + k * 32), idesc,
                      (kb > kb0 || j > 0 || k > 0) ? 1u : 0u);
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
    const int n_local = warp * 32 + lane;
    int part = 0;
    for (int u = u0; u < u1; ++part) {
      const int t = tile_of(u), kb0 = u % KBt;
      const int kb1 = min(KBt, kb0 + (u1 - u));
      u += kb1 - kb0;
      const int buf = part & 1;
      const uint32_t use = (uint32_t)(part >> 1);
      // warp-uniform, then epilogue-uniform decision to go on
      bool ok = !*s_abort && mbar_wait(&tfull[buf], use & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) s_ok[(part & 1) * 4 + warp] = ok ? 1 : 0;
      epi_bar();
      const int pb = (part & 1) * 4;
      if (!(s_ok[pb] && s_ok[pb + 1] && s_ok[pb + 2] && s_ok[pb + 3])) { *s_abort = 1; break; }
      tc_fence_after();
      const int nt = t / p.m_tiles, mt = t % p.m_tiles;
      const int n = nt * TC_BM + n_local;
      const int m0 = mt * NT;
      const int mrows = min(NT, p.M - m0);
      const bool whole = !DUMP && (kb0 == 0 && kb1 == KBt);
      const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(buf * C::NMMA);
      float* wsl = DUMP ? p.ws + (size_t)(t + blockIdx.x) * NT * TC_BM
                        : tc_slot(p.ws, blockIdx.x, part == 0 ? 0 : 1, NT);
#pragma unroll 1
      for (int c0 = 0; c0 < NT; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + c0, v);
        if (SPLIT) {
          float vl[16];
          tmem_ld16(tbase + NT + c0, vl);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] += vl[i];
        }
        if (whole) {
          tc_store_rows<16>(p, m0 + c0, mrows - c0, n, v);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < mrows) wsl[(size_t)(c0 + i) * TC_BM + n_local] = v[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (!DUMP && !whole) {
        __threadfence();
        epi_bar();
        // the tile's contributors: split positions first..last (CTA
        // first * m_tiles + mt_fix .. with m-tile groups)
        const int vt0 = grp ? (t / p.m_tiles) * KBt : t * KBt;   // its first virtual unit
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
          // 8 rows x 8 contributors of loads are issued before any add; the
          // adds run in CTA order (deterministic)
#pragma unroll 1
          for (int m = 0; m < mrows; m += 8) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll 1
            for (int i0 = first; i0 <= last; i0 += 8) {
              float v[8][8];
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const int i = i0 + c;
                const float* src = nullptr;
                if (i <= last) {
                  const int slot = (sk_start(i, vunits, nsplit) >= vt0) ? 0 : 1;
                  const int cta = grp ? i * p.m_tiles + mt_fix : i;
                  src = tc_slot(p.ws, cta, slot, NT) + (size_t)m * TC_BM + n_local;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  v[c][j] = (src && m + j < mrows) ? __ldcg(src + (size_t)j * TC_BM) : 0.f;
              }
#pragma unroll
              for (int c = 0; c < 8; ++c)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] += v[c][j];
            }
            tc_store_rows<8>(p, m0 + m, mrows - m, n, acc);
          }
        }
        epi_bar();   // s_last is reused by the next cut part
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*s_abort && threadIdx.x == 0) raise_status(p.status, ST_GEMM_TIMEOUT);
  if (DUMP) dep_signal_synced(p.done);   // every part of this CTA is stored
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS));
  }
}

}  // namespace uno
