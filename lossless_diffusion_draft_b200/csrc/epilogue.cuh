// Epilogue kernels of the per-layer GEMMs (DUMP-mode tensor-core GEMM).
//
// Each decoder layer is four weight streams - q|k|v, o, gate|up, down - and
// each GEMM leaves fp32 parts of its output tiles in slots (see gemm_tc.cuh).
// The kernel after it adds a tile's parts in CTA order and fuses everything
// up to the next GEMM's input:
//
//   epi_qkv_kernel     q|k|v: LoRA-B, RMSNorm scale, RoPE; q -> attention
//                      input, k and v -> paged KV pool;
//   epi_resid_kernel   o or down: LoRA-B, residual add into x, and the next
//                      RMSNorm's input g * x (bf16 hi/lo rows) with per-tile
//                      sums of squares of x;
//   epi_swiglu_kernel  gate|up: LoRA-B, RMSNorm scale, silu(gate) * up.
//
// RMSNorm (Qwen3-style pre-norm: x / sqrt(mean(x^2) + eps) * g) is split
// around the GEMM: the GEMM reads g * x and the epilogue multiplies its
// output row by 1 / sqrt(mean(x^2) + eps), which is the same product
// (the scale is per token row, i.e. per output row of the projection).
//
// Gated LoRA (summary page "通过离散扩散实现 LLM 无损加速：扩散增强自回归模型",
// section 方法关键点; blog page "…Uno 的无损加速之路", section Diffusion
// Distillation：一步蒸馏 + 块级扩散): y = W x + gate * (alpha / r) * B (A x).
// The GEMM streams the A matrices as extra output tiles next to W, so the
// rank-r product U = A (g * x) comes out of the same pass; the epilogue
// multiplies U by the rows of B (a small tensor-core product per CTA, below)
// and gates it per row.
//
// One CTA takes one 128-column tile of the output (two for SwiGLU) and a
// group of rows (Geo below); a few slot threads share a column, each with a
// few of the rows.  Every load a thread needs is issued before the first
// use, so a CTA costs about one memory round trip.
#pragma once

#include "gemm_tc.cuh"
#include "layers.cuh"

namespace uno {

constexpr int EPI_R = TC_BM;         // LoRA rank the fused epilogue takes (one U tile)

// Where a DUMP-mode GEMM left its parts.
struct PartView {
  const float* ws;                   // slots [tiles + grid][NT][128] fp32
  int NT, units, grid, KBt, m_tiles;
};

// Gated LoRA-B of the epilogue.
struct LoraEpi {
  const bf16* Bl[3];                 // B of each segment [n_seg, r]
  int seg_n0[3];                     // first output column of each segment
  int nseg;
  int u_tile0;                       // n-tile of segment 0's U; segment s at u_tile0 + s
  const float* row_gate;             // [M] gate * alpha / r per row (0: adapter off)
};

struct EpiArgs {
  PartView pv;                       // (prep: NT = M, m_tiles = 1, no parts read)
  int M;
  int lo_off;                        // split rows: lo rows this many rows below (0: none)
  // RMSNorm scale of the GEMM input (null: input not normalised)
  const float* ss;                   // [M][n_ss] sums of squares per 128-column tile
  int n_ss; float d_model, eps;
  int lora; LoraEpi lr;
  // epi_qkv
  f16* q_out; int ld_q;              // rotated q rows, fp16 hi (lo rows lo_off below)
  int H, Hkv, hd;
  const int32_t* row_pos; const int32_t* row_slot;
  const float* cos_t; const float* sin_t; int max_pos;
  KvLayout kv; int layer;
  // epi_resid
  float* x; int d;
  const bf16* g_next;                // next RMSNorm gain (null: no next input)
  bf16* xn; int ld_xn;               // next GEMM input g * x (hi rows; lo rows lo_off below)
  float* ss_out;                     // [M][d / 128]
  int prep;                          // 1: no GEMM parts (layer-0 input preparation)
  // epi_swiglu
  int F; bf16* h;                    // [M][F] (lo rows lo_off below)
  int32_t* status;
  unsigned* done;                    // completion counter the next kernel waits on (or null)
  // completion counter of the GEMM whose parts this kernel reads (null:
  // pdl_wait instead), its CTA count and how long to poll it
  const unsigned* dep; unsigned dep_count;
  unsigned long long dep_limit_ns;
};

// Wait for the GEMM's parts: one thread polls its completion counter and the
// CTA meets it at a barrier (CTA-uniform call), or, without a counter, the
// grid dependency.
__device__ __forceinline__ void epi_wait(const EpiArgs& a) {
  if (a.dep) {
    if (threadIdx.x == 0 && !dep_wait(a.dep, a.dep_count, a.dep_limit_ns))
      raise_status(a.status, ST_DEP_TIMEOUT);
    __syncthreads();
  } else {
    pdl_wait();
  }
}

// Thread layout of an epilogue CTA: NQ row slots x 128 columns, the NQ
// slot threads of a column in adjacent lanes (thread t: slot q = t % NQ,
// column t / NQ).  A thread owns rows j = q + NQ s (s < RPT) of the CTA's RG
// rows.  The LoRA-B dot of a column is split by rank over its slot threads,
// whose partials meet in a fixed shuffle butterfly.
constexpr int EPI_MAX_SS = 64;        // d_model <= 64 * 128
template <int RG_, int NQ_>
struct Geo {
  static constexpr int RG = RG_, NQ = NQ_;
  static constexpr int RPT = (RG + NQ - 1) / NQ;
  static constexpr int THREADS = NQ * TC_BM;
  // LoRA-B tiles: 16 MMA rows, eight warps of 16 columns
  static_assert(RG <= 16 && THREADS == 256, "row group fits one MMA tile; 8 warps x 16 columns");
  static constexpr int KQ = EPI_R / NQ;                     // rank columns per slot thread
  static constexpr int SS_PT = (RG * EPI_MAX_SS + THREADS - 1) / THREADS;
};
typedef Geo<9, 2> GeoQkv;     // 17-row draft pass: two row groups
typedef Geo<9, 2> GeoResid;   // its row groups only: the residual kernel has a 16-byte unit layout

// Row groups never straddle an m-tile of the GEMM (the part slots are per
// m-tile): blockIdx.y = m-tile * groups_per_tile + group.  Returns false for
// a group past the rows (whole CTA).
__host__ __device__ __forceinline__ int epi_groups_per_tile(int NT, int M, int RG) {
  return ((NT < M ? NT : M) + RG - 1) / RG;
}
template <class G>
__device__ __forceinline__ bool row_group(const EpiArgs& a, int* m0, int* nrows) {
  const int gpt = epi_groups_per_tile(a.pv.NT, a.M, G::RG);
  const int mt = blockIdx.y / gpt, g = blockIdx.y % gpt;
  *m0 = mt * a.pv.NT + g * G::RG;
  const int end = min(a.M, (mt + 1) * a.pv.NT);
  *nrows = min(G::RG, end - *m0);
  return *nrows > 0;
}

// Parts of column col of output tile nt for the thread's rows (m0 + q + NQ s).
// part_issue loads the first C contributors (issued before any use);
// part_add adds them in CTA order, the first contributor's part first, then
// reads any further contributors C at a time.
template <class G, int C>
struct PartLoad {
  float x[C][G::RPT];
  int first, last, slot;             // slot: floats between contributors' parts
  const float* base;
};
template <class G, int C>
__device__ __forceinline__ void part_issue(const PartView& v, int nt, int m0, int nrows, int col,
                                           int q, PartLoad<G, C>& L) {
  const int mt = m0 / v.NT;
  const int t = nt * v.m_tiles + mt;
  L.first = sk_owner(t * v.KBt, v.units, v.grid);
  L.last = sk_owner(t * v.KBt + v.KBt - 1, v.units, v.grid);
  L.slot = v.NT * TC_BM;
  L.base = v.ws + ((size_t)t * v.NT + (m0 - mt * v.NT) + q) * TC_BM + col;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const int i = L.first + c;
#pragma unroll
    for (int s = 0; s < G::RPT; ++s)
      L.x[c][s] = (i <= L.last && q + G::NQ * s < nrows)
                      ? __ldcg(L.base + (size_t)i * L.slot + (size_t)(G::NQ * s) * TC_BM) : 0.f;
  }
}
template <class G, int C>
__device__ __forceinline__ void part_add(PartLoad<G, C>& L, int nrows, int q, float (&acc)[G::RPT]) {
#pragma unroll
  for (int s = 0; s < G::RPT; ++s) acc[s] = 0.f;
  for (int i0 = L.first;; i0 += C) {
#pragma unroll
    for (int c = 0; c < C; ++c)
#pragma unroll
      for (int s = 0; s < G::RPT; ++s) acc[s] += L.x[c][s];
    if (i0 + C > L.last) break;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int i = i0 + C + c;
#pragma unroll
      for (int s = 0; s < G::RPT; ++s)
        L.x[c][s] = (i <= L.last && q + G::NQ * s < nrows)
                        ? __ldcg(L.base + (size_t)i * L.slot + (size_t)(G::NQ * s) * TC_BM) : 0.f;
    }
  }
}

// Sums of squares of rows m0 .. m0 + nrows (all n_ss tiles of each): the
// (row, tile) values are spread over the CTA's threads, all loads issued
// together.
template <class G>
struct SsLoad { float v[G::SS_PT]; };
template <class G>
__device__ __forceinline__ void ss_issue(const EpiArgs& a, int m0, int nrows, SsLoad<G>& L) {
#pragma unroll
  for (int k = 0; k < G::SS_PT; ++k) {
    const int e = threadIdx.x + k * G::THREADS;
    L.v[k] = (a.ss && e < nrows * a.n_ss) ? __ldcg(a.ss + (size_t)m0 * a.n_ss + e) : 0.f;
  }
}
// 1 / sqrt(mean(x^2) + eps) per row into s_inv (tiles added in tile order);
// 1 without a norm.  Syncs the CTA (twice).
template <class G>
__device__ __forceinline__ void ss_finish(const EpiArgs& a, int nrows, const SsLoad<G>& L,
                                          float* s_ss, float* s_inv) {
#pragma unroll
  for (int k = 0; k < G::SS_PT; ++k) {
    const int e = threadIdx.x + k * G::THREADS;
    if (e < nrows * a.n_ss) s_ss[e] = L.v[k];
  }
  __syncthreads();
  const int j = threadIdx.x;
  if (j < G::RG) {
    float inv = 1.f;
    if (a.ss && j < nrows) {
      float t = 0.f;
      for (int i = 0; i < a.n_ss; ++i) t += s_ss[j * a.n_ss + i];
      inv = 1.0f / sqrtf(t / a.d_model + a.eps);
    }
    s_inv[j] = inv;
  }
  __syncthreads();
}

// Segment of output column n.
__device__ __forceinline__ int lora_seg(const LoraEpi& lr, int n) {
  int s = 0;
  for (int k = 1; k < lr.nseg; ++k)
    if (n >= lr.seg_n0[k]) s = k;
  return s;
}

// ---------------------------------------------------------------------------
// LoRA-B on the tensor cores: dot[j][c] = sum_k U[j][k] B[c][k] for the
// CTA's rows j (at most 16) and 128 columns c, as mma.sync m16n8k16 (bf16
// in, fp32 accumulate) with U fed as a bf16 hi/lo pair (~16 mantissa bits,
// like the GEMM inputs) and B, a bf16 weight, exact.  Warp w takes the
// columns 16 w .. 16 w + 15 (two n-tiles of 8).  The rank order inside a
// k-step is free as long as U and B agree: in k-step s, thread t of a quad
// puts ranks 32 t + 4 s + {0, 1} in the k-slots {2t, 2t+1} and
// 32 t + 4 s + {2, 3} in {2t+8, 2t+9}.  Its B values for its column are then
// the 32 contiguous ranks 32 t .. 32 t + 31 (four 16-byte loads per n-tile,
// issued before the dependency wait), and its U values of a row are 8
// contiguous bf16 per pair of k-steps (one 16-byte shared-memory load).
// ---------------------------------------------------------------------------
constexpr int EPI_UP = EPI_R + 8;   // row pitch of the bf16 U tiles: 272 B, conflict-free loads
static_assert(EPI_R == 128, "the k-step rank order covers 128 ranks");

struct BFrag { uint4 b[2][4]; };    // [n-tile][16-byte piece of the thread's 32 ranks]
// col0: the adapter row (segment column) of the warp's first column
__device__ __forceinline__ void bfrag_issue(const EpiArgs& a, int seg, int col0, BFrag& B) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const uint4* src =
        reinterpret_cast<const uint4*>(a.lr.Bl[seg] + (size_t)(col0 + 8 * nt + g) * EPI_R + 32 * t);
#pragma unroll
    for (int e = 0; e < 4; ++e) B.b[nt][e] = __ldg(src + e);
  }
}
// The same bytes into L2 only (one prefetch per thread and n-tile: 64 bytes).
__device__ __forceinline__ void bfrag_prefetch(const EpiArgs& a, int seg, int col0) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.lr.Bl[seg] + (size_t)(col0 + 8 * nt + g) * EPI_R + 32 * t));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The dots of the CTA's first `rows` rows into sDot[row][128].  sUh / sUl
// ([16][EPI_UP] bf16) must be complete (caller syncs); rows past `rows`
// may hold anything (an MMA row depends only on its own U row).
__device__ __forceinline__ void lora_mma(const BFrag& B, const bf16* sUh, const bf16* sUl,
                                         float* sDot, int rows) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int s2 = 0; s2 < 4; ++s2) {
    const int o = 32 * t + 8 * s2;   // ranks 32 t + 8 s2 .. + 7: k-steps 2 s2 and 2 s2 + 1
    const uint4 h0 = *reinterpret_cast<const uint4*>(sUh + g * EPI_UP + o);
    const uint4 h1 = *reinterpret_cast<const uint4*>(sUh + (g + 8) * EPI_UP + o);
    const uint4 l0 = *reinterpret_cast<const uint4*>(sUl + g * EPI_UP + o);
    const uint4 l1 = *reinterpret_cast<const uint4*>(sUl + (g + 8) * EPI_UP + o);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int ks = 2 * s2 + half;
      // A registers: (row g, slots 2t..), (row g+8, 2t..), (row g, 2t+8..), (row g+8, 2t+8..)
      const uint32_t ah[4] = {half ? h0.z : h0.x, half ? h1.z : h1.x, half ? h0.w : h0.y,
                              half ? h1.w : h1.y};
      const uint32_t al[4] = {half ? l0.z : l0.x, half ? l1.z : l1.x, half ? l0.w : l0.y,
                              half ? l1.w : l1.y};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const uint4 bb = B.b[nt][ks >> 1];
        const uint32_t b0 = (ks & 1) ? bb.z : bb.x, b1 = (ks & 1) ? bb.w : bb.y;
        mma_bf16_16816(d[nt], ah, b0, b1);
        mma_bf16_16816(d[nt], al, b0, b1);
      }
    }
  }
  // accumulator: (row g, columns 2t, 2t+1) and (row g+8, the same columns)
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int c = 16 * warp + 8 * nt + 2 * t;
    if (g < rows) {
      sDot[g * TC_BM + c] = d[nt][0];
      sDot[g * TC_BM + c + 1] = d[nt][1];
    }
    if (g + 8 < rows) {
      sDot[(g + 8) * TC_BM + c] = d[nt][2];
      sDot[(g + 8) * TC_BM + c + 1] = d[nt][3];
    }
  }
}

// acc += gate * dot for the thread's rows of column col (sDot complete:
// caller syncs).
template <class G>
__device__ __forceinline__ void lora_add(const float* sDot, int col, int q, int nrows,
                                         const float (&gate)[G::RPT], float (&acc)[G::RPT]) {
#pragma unroll
  for (int s = 0; s < G::RPT; ++s) {
    const int j = q + G::NQ * s;
    if (j < nrows) acc[s] += gate[s] * sDot[j * TC_BM + col];
  }
}

// The U tile of segment seg, column (rank) col, the thread's rows: loads,
// then the sums as a bf16 hi/lo pair into sUh / sUl [16][EPI_UP].  The
// caller syncs before they are read.
template <class G, int C>
__device__ __forceinline__ void u_issue(const EpiArgs& a, int seg, int m0, int nrows, int col, int q,
                                        PartLoad<G, C>& L) {
  part_issue(a.pv, a.lr.u_tile0 + seg, m0, nrows, col, q, L);
}
template <class G, int C>
__device__ __forceinline__ void u_store(PartLoad<G, C>& L, int nrows, int col, int q, bf16* sUh,
                                        bf16* sUl) {
  float u[G::RPT];
  part_add(L, nrows, q, u);
#pragma unroll
  for (int s = 0; s < G::RPT; ++s) {
    const int j = q + G::NQ * s;
    if (j < nrows) {
      const bf16 h = from_f<bf16>(u[s]);
      sUh[j * EPI_UP + col] = h;
      sUl[j * EPI_UP + col] = from_f<bf16>(u[s] - to_f(h));
    }
  }
}

// Row gates of the thread's rows (0 past M).
template <class G>
__device__ __forceinline__ void gate_issue(const EpiArgs& a, int m0, int nrows, int q,
                                           float (&g)[G::RPT]) {
#pragma unroll
  for (int s = 0; s < G::RPT; ++s)
    g[s] = q + G::NQ * s < nrows ? __ldcg(a.lr.row_gate + m0 + q + G::NQ * s) : 0.f;
}

// ---------------------------------------------------------------------------
// q|k|v: grid ((H + 2 Hkv) hd / 128, row groups), GeoQkv::THREADS threads.
// ---------------------------------------------------------------------------
// At most 128 registers a thread: two of its warps and two attention warps
// (128 each) fill one SM sub-partition's 16,384 registers, so the attention
// starts beside this kernel.
__global__ void __maxnreg__(128) epi_qkv_kernel(const EpiArgs a) {
  typedef GeoQkv G;
  constexpr int C = 4;
  __shared__ float s_inv[G::RG];
  __shared__ float s_ss[G::RG * EPI_MAX_SS];
  __shared__ __align__(16) bf16 sUh[16 * EPI_UP];
  __shared__ __align__(16) bf16 sUl[16 * EPI_UP];
  __shared__ float sY[G::RG][TC_BM];          // LoRA dots first, then the rows for RoPE
  pdl_trigger();
  const int nt = blockIdx.x;
  int m0, nrows;
  if (!row_group<G>(a, &m0, &nrows)) { dep_signal(a.done); return; }
  const int q = threadIdx.x % G::NQ, col = threadIdx.x / G::NQ;
  const int n = nt * TC_BM + col;
  const int qcols = a.H * a.hd, kcols = a.Hkv * a.hd;
  const int half = a.hd / 2;
  const int hi = n % a.hd;                 // index inside the head
  const bool rot = n < qcols + kcols;      // q and k are rotated, v is not
  const bool kv_tile = n >= qcols;
  const int ci = hi < half ? hi : hi - half;
  // the adapter rows are weights: read while the GEMM before is still running
  const int seg = a.lora ? lora_seg(a.lr, nt * TC_BM) : 0;
  BFrag B;
  if (a.lora) bfrag_issue(a, seg, nt * TC_BM + 16 * (threadIdx.x >> 5) - a.lr.seg_n0[seg], B);
  // The row tables, the row gates and the page table are complete before
  // this kernel starts (the pass's first kernel after build_rows waits for
  // it before letting the next one launch): positions, slots, RoPE entries
  // and KV pages are fetched while the GEMM before still runs.  Loads before
  // the wait bypass L1 (ld.global.cg), which may still hold lines of an
  // earlier pass until the dependency wait.
  int pos[G::RPT], slot[G::RPT];
#pragma unroll
  for (int s = 0; s < G::RPT; ++s) {
    const int j = q + G::NQ * s;
    pos[s] = j < nrows ? __ldcg(a.row_pos + m0 + j) : 0;
    slot[s] = (j < nrows && kv_tile) ? __ldcg(a.row_slot + m0 + j) : 0;
  }
  float gate[G::RPT];
  if (a.lora) gate_issue<G>(a, m0, nrows, q, gate);
  float cs[G::RPT], sn[G::RPT];
  int page[G::RPT], pok[G::RPT];
#pragma unroll
  for (int s = 0; s < G::RPT; ++s) {
    const int j = q + G::NQ * s;
    const int pc = (pos[s] >= 0 && pos[s] < a.max_pos) ? pos[s] : 0;
    cs[s] = rot ? a.cos_t[(size_t)pc * half + ci] : 0.f;
    sn[s] = rot ? a.sin_t[(size_t)pc * half + ci] : 0.f;
    int ok = 0;
    page[s] = (j < nrows && kv_tile) ? a.kv.page_of(slot[s], pos[s], ok) : 0;
    pok[s] = ok;
  }
  epi_wait(a);

  // ---- every load of what the GEMM (and the residual kernel before it) wrote
  SsLoad<G> ssv;
  ss_issue(a, m0, nrows, ssv);
  PartLoad<G, C> LU, LP;
  if (a.lora) u_issue(a, seg, m0, nrows, col, q, LU);
  part_issue(a.pv, nt, m0, nrows, col, q, LP);

  // ---- then the arithmetic
  if (a.lora) u_store(LU, nrows, col, q, sUh, sUl);
  ss_finish(a, nrows, ssv, s_ss, s_inv);     // syncs: sUh / sUl complete too
  float acc[G::RPT];
  part_add(LP, nrows, q, acc);
  if (a.lora) {
    lora_mma(B, sUh, sUl, &sY[0][0], nrows);
    __syncthreads();
    // each thread reads the dots of its own (row, column) entries, which
    // only it rewrites below
    lora_add<G>(&sY[0][0], col, q, nrows, gate, acc);
  }
#pragma unroll
  for (int s = 0; s < G::RPT; ++s) {
    const int j = q + G::NQ * s;
    if (j < nrows) sY[j][col] = acc[s] * s_inv[j];
  }
  __syncthreads();

#pragma unroll
  for (int s = 0; s < G::RPT; ++s) {
    const int j = q + G::NQ * s;
    if (j >= nrows) continue;
    const int m = m0 + j;
    const bool ok_pos = pos[s] >= 0 && pos[s] < a.max_pos;
    float y = sY[j][col];
    // rotate-half: (x1, x2) -> (x1 c - x2 s, x2 c + x1 s)
    if (rot) y = hi < half ? sY[j][col] * cs[s] - sY[j][col + half] * sn[s]
                           : sY[j][col] * cs[s] + sY[j][col - half] * sn[s];
    if (n < qcols) {
      // q as an fp16 hi/lo pair (lo rows lo_off below): the attention adds
      // q_hi K + q_lo K
      const f16 qh = from_f<f16>(y);
      a.q_out[(size_t)m * a.ld_q + n] = qh;
      a.q_out[(size_t)(a.lo_off + m) * a.ld_q + n] = from_f<f16>(y - to_f(qh));
    } else {
      const bool is_k = n < qcols + kcols;
      const int head = (n - (is_k ? qcols : qcols + kcols)) / a.hd;
      const size_t off =
          a.kv.offset_in_page(a.layer, page[s], pos[s], is_k ? 0 : a.kv.v_plane(), head) + hi;
      if (pok[s] && ok_pos) {
        f16* pool = reinterpret_cast<f16*>(a.kv.pool);
        const f16 yh = from_f<f16>(y);
        pool[off] = yh;
        if (is_k) pool[off + a.kv.plane_stride()] = from_f<f16>(y - to_f(yh));   // K lo plane
      } else if (hi == 0 && is_k) {
        raise_status(a.status, ST_POS_OVERFLOW);
      }
    }
  }
  dep_signal(a.done);   // q rows and K/V rows stored (the attention waits on it)
}

// ---------------------------------------------------------------------------
// o / down (and, with prep = 1, the layer-0 input): grid (d / 128, row groups
// of GeoResid::RG), RESID_THREADS threads.  Thread t owns one unit: row
// t / 32 of the group and the four columns 4 (t % 32) .. + 3 of the tile, so
// warp w holds row w and every global access is a 16-byte one (a
// contributor's part of the CTA's rows is one contiguous block).  x += y;
// then the next GEMM's input g * x (hi/lo) and the row's sum of squares over
// the tile (a warp reduction).
// ---------------------------------------------------------------------------
constexpr int RESID_THREADS = GeoResid::RG * 32;

// The parts of output tile nt for one unit: contributors issued C at a
// time; part4_add adds them in CTA order.
template <int C>
struct Part4 {
  float4 x[C];
  int first, last, slot;
  const float* base;
};
template <int C>
__device__ __forceinline__ void part4_issue(const PartView& v, int nt, int m0, int j, int c0, bool live,
                                            Part4<C>& L) {
  const int mt = m0 / v.NT;
  const int t = nt * v.m_tiles + mt;
  L.first = sk_owner(t * v.KBt, v.units, v.grid);
  L.last = sk_owner(t * v.KBt + v.KBt - 1, v.units, v.grid);
  L.slot = v.NT * TC_BM;
  L.base = v.ws + ((size_t)t * v.NT + (m0 - mt * v.NT) + j) * TC_BM + c0;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const int i = L.first + c;
    L.x[c] = (live && i <= L.last) ? __ldcg(reinterpret_cast<const float4*>(L.base + (size_t)i * L.slot))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}
template <int C>
__device__ __forceinline__ float4 part4_add(Part4<C>& L, bool live) {
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i0 = L.first;; i0 += C) {
#pragma unroll
    for (int c = 0; c < C; ++c) {
      acc.x += L.x[c].x; acc.y += L.x[c].y; acc.z += L.x[c].z; acc.w += L.x[c].w;
    }
    if (i0 + C > L.last) break;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int i = i0 + C + c;
      L.x[c] = (live && i <= L.last)
                   ? __ldcg(reinterpret_cast<const float4*>(L.base + (size_t)i * L.slot))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  return acc;
}

__global__ void __launch_bounds__(RESID_THREADS) epi_resid_kernel(const EpiArgs a) {
  typedef GeoResid G;
  constexpr int C = 6;
  __shared__ __align__(16) bf16 sUh[16 * EPI_UP];
  __shared__ __align__(16) bf16 sUl[16 * EPI_UP];
  __shared__ __align__(16) float sDot[G::RG * TC_BM];
  // The layer-0 input preparation is the pass's first kernel after
  // build_rows: it lets the next kernel launch only after build_rows has
  // completed, so every later kernel of the pass may read the row tables
  // before its own wait.
  if (a.prep) pdl_wait();
  pdl_trigger();
  const int nt = blockIdx.x;
  int m0, nrows;
  if (!row_group<G>(a, &m0, &nrows)) { dep_signal(a.done); return; }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = warp;                        // the unit's row in the group
  const int c0 = 4 * lane;                   // its first column in the tile
  const int n = nt * TC_BM + c0;
  const bool live = j < nrows;
  const bool lora = !a.prep && a.lora;
  // weights (the next norm's gains, the adapter rows) before the dependency wait
  float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (a.g_next) {
    const uint2 gg = __ldg(reinterpret_cast<const uint2*>(a.g_next + n));
    const __nv_bfloat162 g01 = *reinterpret_cast<const __nv_bfloat162*>(&gg.x);
    const __nv_bfloat162 g23 = *reinterpret_cast<const __nv_bfloat162*>(&gg.y);
    g4 = make_float4(__low2float(g01), __high2float(g01), __low2float(g23), __high2float(g23));
  }
  BFrag B;
  if (lora && warp < 8) bfrag_issue(a, 0, nt * TC_BM + 16 * warp, B);
  // the row gate (build_rows' table, complete before this kernel starts;
  // read through L2: L1 may hold an earlier pass's line before the wait)
  const float gt = (lora && live) ? __ldcg(a.lr.row_gate + m0 + j) : 0.f;
  epi_wait(a);

  // ---- every global load first
  const size_t xi = (size_t)(m0 + j) * a.d + n;
  // through L2, like every load of another kernel's output here: with a
  // completion counter there is no grid wait to drop stale L1 lines
  float4 xv = live ? __ldcg(reinterpret_cast<const float4*>(a.x + xi)) : make_float4(0.f, 0.f, 0.f, 0.f);
  if (!a.prep) {
    Part4<C> LU, LP;
    if (lora) part4_issue(a.pv, a.lr.u_tile0, m0, j, c0, live, LU);
    part4_issue(a.pv, nt, m0, j, c0, live, LP);
    // ---- then the arithmetic
    if (lora) {
      // U's rows as bf16 hi/lo for the tensor-core LoRA-B
      const float4 u = part4_add(LU, live);
      if (live) store4_split(sUh, sUl, (size_t)j * EPI_UP + c0, u);
      __syncthreads();
      if (warp < 8) lora_mma(B, sUh, sUl, sDot, nrows);
    }
    float4 y = part4_add(LP, live);
    if (lora) {
      __syncthreads();
      const float4 dt = *reinterpret_cast<const float4*>(sDot + j * TC_BM + c0);
      y.x += gt * dt.x; y.y += gt * dt.y; y.z += gt * dt.z; y.w += gt * dt.w;
    }
    xv.x += y.x; xv.y += y.y; xv.z += y.z; xv.w += y.w;
    if (live) *reinterpret_cast<float4*>(a.x + xi) = xv;
  }
  if (a.g_next) {
    bf16* lo = a.lo_off ? a.xn + (size_t)a.lo_off * a.ld_xn : nullptr;
    if (live)
      store4_split(a.xn, lo, (size_t)(m0 + j) * a.ld_xn + n,
                   make_float4(g4.x * xv.x, g4.y * xv.y, g4.z * xv.z, g4.w * xv.w));
    float sq = xv.x * xv.x + xv.y * xv.y + xv.z * xv.z + xv.w * xv.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (live && lane == 0) a.ss_out[(size_t)(m0 + j) * (a.d / TC_BM) + nt] = sq;
  }
  dep_signal(a.done);
}

// ---------------------------------------------------------------------------
// gate|up -> silu(gate) * up: grid (F / 128, row groups of GeoResid::RG),
// RESID_THREADS threads in the residual kernel's unit layout: thread t owns
// row t / 32 of the group and features 4 (t % 32) .. + 3 of the tile, so every
// part, U and output access is one 16-byte access per contributor and the
// row's RMSNorm scale is a warp reduction of its per-tile sums.  Gate's
// adapter runs first (its rows in registers since before the dependency
// wait), up's after it (prefetched into L2 meanwhile); both through the
// same shared U tile.  Two CTAs per SM: the decode passes' 2 x F / 128 CTAs
// are one wave.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(RESID_THREADS, 2) epi_swiglu_kernel(const EpiArgs a) {
  typedef GeoResid G;
  constexpr int C = 2;
  __shared__ __align__(16) bf16 sUh[16 * EPI_UP];
  __shared__ __align__(16) bf16 sUl[16 * EPI_UP];
  __shared__ __align__(16) float sDot[G::RG * TC_BM];
  pdl_trigger();
  const int ft = blockIdx.x;
  int m0, nrows;
  if (!row_group<G>(a, &m0, &nrows)) { dep_signal(a.done); return; }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = warp;                        // the unit's row in the group
  const int c0 = 4 * lane;                   // its first feature in the tile
  const int f = ft * TC_BM + c0;
  const bool live = j < nrows;
  const int ut = a.F / TC_BM + ft;           // the up tile of the same features
  const bool lora = a.lora != 0;
  // adapter rows are weights: gate's into registers and up's into L2 while
  // the GEMM before is still running
  BFrag B;
  const int fw = ft * TC_BM + 16 * warp;     // the warp's first feature (warps 0-7)
  if (lora && warp < 8) {
    bfrag_issue(a, 0, fw, B);
    bfrag_prefetch(a, 1, fw);
  }
  // the row gate (build_rows' table, complete before this kernel starts;
  // read through L2: L1 may hold an earlier pass's line before the wait)
  const float gt = (lora && live) ? __ldcg(a.lr.row_gate + m0 + j) : 0.f;
  epi_wait(a);

  // ---- every global load first
  float ss0 = 0.f, ss1 = 0.f;
  if (a.ss && live) {
    const float* sr = a.ss + (size_t)(m0 + j) * a.n_ss;
    if (lane < a.n_ss) ss0 = __ldcg(sr + lane);
    if (lane + 32 < a.n_ss) ss1 = __ldcg(sr + lane + 32);
  }
  Part4<C> LG, LUp, L0, L1;
  part4_issue(a.pv, ft, m0, j, c0, live, LG);
  part4_issue(a.pv, ut, m0, j, c0, live, LUp);
  if (lora) {
    part4_issue(a.pv, a.lr.u_tile0, m0, j, c0, live, L0);
    part4_issue(a.pv, a.lr.u_tile0 + 1, m0, j, c0, live, L1);
  }
  // ---- then the arithmetic
  float inv = 1.f;
  if (a.ss) {
    float t = ss0 + ss1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    inv = 1.0f / sqrtf(t / a.d_model + a.eps);
  }
  if (lora) {
    const float4 u = part4_add(L0, live);
    if (live) store4_split(sUh, sUl, (size_t)j * EPI_UP + c0, u);
    __syncthreads();
    if (warp < 8) lora_mma(B, sUh, sUl, sDot, nrows);
  }
  float4 g = part4_add(LG, live);
  float4 u = part4_add(LUp, live);
  if (lora) {
    if (warp < 8) bfrag_issue(a, 1, fw, B);
    const float4 u1 = part4_add(L1, live);
    __syncthreads();                         // gate's dots complete, U tile free
    const float4 dg = *reinterpret_cast<const float4*>(sDot + j * TC_BM + c0);
    g.x += gt * dg.x; g.y += gt * dg.y; g.z += gt * dg.z; g.w += gt * dg.w;
    if (live) store4_split(sUh, sUl, (size_t)j * EPI_UP + c0, u1);
    __syncthreads();                         // every thread read its gate dots
    if (warp < 8) lora_mma(B, sUh, sUl, sDot, nrows);
    __syncthreads();
    const float4 du = *reinterpret_cast<const float4*>(sDot + j * TC_BM + c0);
    u.x += gt * du.x; u.y += gt * du.y; u.z += gt * du.z; u.w += gt * du.w;
  }
  if (live) {
    float4 h;
    const float gx = g.x * inv, gy = g.y * inv, gz = g.z * inv, gw = g.w * inv;
    h.x = gx / (1.0f + expf(-gx)) * (u.x * inv);
    h.y = gy / (1.0f + expf(-gy)) * (u.y * inv);
    h.z = gz / (1.0f + expf(-gz)) * (u.z * inv);
    h.w = gw / (1.0f + expf(-gw)) * (u.w * inv);
    bf16* lo = a.lo_off ? a.h + (size_t)a.lo_off * a.F : nullptr;
    store4_split(a.h, lo, (size_t)(m0 + j) * a.F + f, h);
  }
  dep_signal(a.done);
}

}  // namespace uno
