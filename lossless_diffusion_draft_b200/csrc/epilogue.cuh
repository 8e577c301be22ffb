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
// multiplies U by the rows of B on the CUDA cores (r MACs per output) and
// gates it per row.
//
// One CTA takes one 128-column tile of the output (two for SwiGLU) and
// EPI_RG rows; a thread owns one column.  Every load a thread needs is issued before the first use,
// so a CTA costs about one memory round trip.
#pragma once

#include "gemm_tc.cuh"
#include "layers.cuh"

namespace uno {

constexpr int EPI_RG = 9;            // token rows per CTA (a 17-row draft pass: two groups)
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
  bf16* q_out; int ld_q;
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
};

// Parts of tile column col of output tile nt, rows m0 .. m0 + nrows.
// part_issue loads the first C contributors (issued before any use);
// part_add adds them in CTA order, the first contributor's part first, then
// reads any further contributors C at a time.
// Row groups never straddle an m-tile of the GEMM (the part slots are per
// m-tile): blockIdx.y = m-tile * groups_per_tile + group.  Returns false for
// a group past the rows (whole CTA).
__host__ __device__ __forceinline__ int epi_groups_per_tile(int NT, int M) {
  return ((NT < M ? NT : M) + EPI_RG - 1) / EPI_RG;
}
__device__ __forceinline__ bool row_group(const EpiArgs& a, int* m0, int* nrows) {
  const int gpt = epi_groups_per_tile(a.pv.NT, a.M);
  const int mt = blockIdx.y / gpt, g = blockIdx.y % gpt;
  *m0 = mt * a.pv.NT + g * EPI_RG;
  const int end = min(a.M, (mt + 1) * a.pv.NT);
  *nrows = min(EPI_RG, end - *m0);
  return *nrows > 0;
}

template <int C>
struct PartLoad {
  float x[C][EPI_RG];
  int first, last;
  const float* base; size_t slot;
};
template <int C>
__device__ __forceinline__ void part_issue(const PartView& v, int nt, int m0, int nrows, int col,
                                           PartLoad<C>& L) {
  const int mt = m0 / v.NT;
  const int t = nt * v.m_tiles + mt;
  L.first = sk_owner(t * v.KBt, v.units, v.grid);
  L.last = sk_owner(t * v.KBt + v.KBt - 1, v.units, v.grid);
  L.slot = (size_t)v.NT * TC_BM;
  L.base = v.ws + ((size_t)t * v.NT + (m0 - mt * v.NT)) * TC_BM + col;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    const int i = L.first + c;
#pragma unroll
    for (int j = 0; j < EPI_RG; ++j)
      L.x[c][j] = (i <= L.last && j < nrows) ? __ldcg(L.base + (size_t)i * L.slot + (size_t)j * TC_BM)
                                              : 0.f;
  }
}
template <int C>
__device__ __forceinline__ void part_add(PartLoad<C>& L, int nrows, float (&acc)[EPI_RG]) {
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) acc[j] = 0.f;
  for (int i0 = L.first;; i0 += C) {
#pragma unroll
    for (int c = 0; c < C; ++c)
#pragma unroll
      for (int j = 0; j < EPI_RG; ++j) acc[j] += L.x[c][j];
    if (i0 + C > L.last) break;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int i = i0 + C + c;
#pragma unroll
      for (int j = 0; j < EPI_RG; ++j)
        L.x[c][j] = (i <= L.last && j < nrows)
                        ? __ldcg(L.base + (size_t)i * L.slot + (size_t)j * TC_BM) : 0.f;
    }
  }
}

// Sums of squares of rows m0 .. m0 + nrows (all tiles): one load per
// (row, tile) by threads 0..127, all issued together.
constexpr int EPI_MAX_SS = 64;        // d_model <= 64 * 128
__device__ __forceinline__ void ss_issue(const EpiArgs& a, int m0, int nrows, float (&v)[4]) {
  const int n = nrows * a.n_ss;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = threadIdx.x + k * TC_BM;
    v[k] = (a.ss && threadIdx.x < TC_BM && e < n) ? __ldcg(a.ss + (size_t)m0 * a.n_ss + e) : 0.f;
  }
}
// 1 / sqrt(mean(x^2) + eps) per row into s_inv (tiles added in tile order);
// 1 without a norm.  Call with the values of ss_issue; syncs the CTA.
__device__ __forceinline__ void ss_finish(const EpiArgs& a, int nrows, const float (&v)[4],
                                          float* s_ss, float* s_inv) {
  const int n = nrows * a.n_ss;
  if (threadIdx.x < TC_BM) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = threadIdx.x + k * TC_BM;
      if (e < n) s_ss[e] = v[k];
    }
  }
  __syncthreads();
  const int j = threadIdx.x;
  if (j < EPI_RG) {
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

// One B row of the adapter (EPI_R bf16), loaded whole.
struct BRow { uint4 b[EPI_R / 8]; };
__device__ __forceinline__ void brow_issue(const EpiArgs& a, int s, int nb, BRow& B) {
  const uint4* src = reinterpret_cast<const uint4*>(a.lr.Bl[s] + (size_t)nb * EPI_R);
#pragma unroll
  for (int e = 0; e < EPI_R / 8; ++e) B.b[e] = __ldg(src + e);
}

// acc[j] += gate[j] * sum_k sU[j][k] B[k].
__device__ __forceinline__ void lora_dot(const BRow& B, const float* sU, const float (&gate)[EPI_RG],
                                         float (&acc)[EPI_RG]) {
  float dot[EPI_RG];
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) dot[j] = 0.f;
#pragma unroll
  for (int e = 0; e < EPI_R / 8; ++e) {
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&B.b[e]);
    float bf[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      bf[2 * h] = __low2float(b2[h]);
      bf[2 * h + 1] = __high2float(b2[h]);
    }
#pragma unroll
    for (int j = 0; j < EPI_RG; ++j) {
      const float4* u4 = reinterpret_cast<const float4*>(sU + j * EPI_R + e * 8);
      const float4 x0 = u4[0], x1 = u4[1];
      dot[j] += x0.x * bf[0] + x0.y * bf[1] + x0.z * bf[2] + x0.w * bf[3] + x1.x * bf[4] +
                x1.y * bf[5] + x1.z * bf[6] + x1.w * bf[7];
    }
  }
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) acc[j] += gate[j] * dot[j];
}

// The U tile of segment s (column col of its EPI_R rank columns): loads, then
// its sums into sU[EPI_RG][EPI_R].  The caller syncs before sU is read.
template <int C>
__device__ __forceinline__ void u_issue(const EpiArgs& a, int s, int m0, int nrows, int col,
                                        PartLoad<C>& L) {
  part_issue(a.pv, a.lr.u_tile0 + s, m0, nrows, col, L);
}
template <int C>
__device__ __forceinline__ void u_store(PartLoad<C>& L, int nrows, int col, float* sU) {
  float u[EPI_RG];
  part_add(L, nrows, u);
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) sU[j * EPI_R + col] = u[j];
}

// Row gates of the CTA's rows (0 past M).
__device__ __forceinline__ void gate_issue(const EpiArgs& a, int m0, int nrows, float (&g)[EPI_RG]) {
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) g[j] = j < nrows ? __ldg(a.lr.row_gate + m0 + j) : 0.f;
}

// ---------------------------------------------------------------------------
// q|k|v: grid ((H + 2 Hkv) hd / 128, ceil(M / EPI_RG)), 128 threads.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(TC_BM) epi_qkv_kernel(const EpiArgs a) {
  constexpr int C = 4;
  __shared__ float s_inv[EPI_RG];
  __shared__ float s_ss[EPI_RG * EPI_MAX_SS];
  __shared__ __align__(16) float sU[EPI_RG * EPI_R];
  __shared__ float sY[EPI_RG][TC_BM];
  pdl_trigger();
  pdl_wait();
  const int nt = blockIdx.x;
  int m0, nrows;
  if (!row_group(a, &m0, &nrows)) return;
  const int i = threadIdx.x;
  const int n = nt * TC_BM + i;
  const int qcols = a.H * a.hd, kcols = a.Hkv * a.hd;
  const int half = a.hd / 2;
  const int hi = n % a.hd;                 // index inside the head
  const bool rot = n < qcols + kcols;      // q and k are rotated, v is not
  const int ci = hi < half ? hi : hi - half;

  // ---- every global load first
  const bool kv_tile = n >= qcols;
  int pos[EPI_RG], slot[EPI_RG];
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) {
    pos[j] = j < nrows ? a.row_pos[m0 + j] : 0;
    slot[j] = (j < nrows && kv_tile) ? a.row_slot[m0 + j] : 0;
  }
  float ssv[4];
  ss_issue(a, m0, nrows, ssv);
  const int s = a.lora ? lora_seg(a.lr, nt * TC_BM) : 0;
  PartLoad<C> LU, LP;
  BRow B;
  float gate[EPI_RG];
  if (a.lora) {
    u_issue(a, s, m0, nrows, i, LU);
    brow_issue(a, s, n - a.lr.seg_n0[s], B);
    gate_issue(a, m0, nrows, gate);
  }
  part_issue(a.pv, nt, m0, nrows, i, LP);
  // second round, addressed by the rows' positions and slots: RoPE table
  // entries and the KV pages
  float cs[EPI_RG], sn[EPI_RG];
  int page[EPI_RG], pok[EPI_RG];
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) {
    const int pc = (pos[j] >= 0 && pos[j] < a.max_pos) ? pos[j] : 0;
    cs[j] = rot ? a.cos_t[(size_t)pc * half + ci] : 0.f;
    sn[j] = rot ? a.sin_t[(size_t)pc * half + ci] : 0.f;
    int ok = 0;
    page[j] = (j < nrows && kv_tile) ? a.kv.page_of(slot[j], pos[j], ok) : 0;
    pok[j] = ok;
  }

  // ---- then the arithmetic
  if (a.lora) u_store(LU, nrows, i, sU);
  ss_finish(a, nrows, ssv, s_ss, s_inv);     // syncs: sU complete too
  float acc[EPI_RG];
  part_add(LP, nrows, acc);
  if (a.lora) lora_dot(B, sU, gate, acc);
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) sY[j][i] = acc[j] * s_inv[j];
  __syncthreads();

#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) {
    if (j >= nrows) continue;
    const int m = m0 + j;
    const bool ok_pos = pos[j] >= 0 && pos[j] < a.max_pos;
    float y = sY[j][i];
    // rotate-half: (x1, x2) -> (x1 c - x2 s, x2 c + x1 s)
    if (rot) y = hi < half ? sY[j][i] * cs[j] - sY[j][i + half] * sn[j]
                           : sY[j][i] * cs[j] + sY[j][i - half] * sn[j];
    if (n < qcols) {
      a.q_out[(size_t)m * a.ld_q + n] = from_f<bf16>(y);
    } else {
      const bool is_k = n < qcols + kcols;
      const int head = (n - (is_k ? qcols : qcols + kcols)) / a.hd;
      const size_t off = a.kv.offset_in_page(a.layer, page[j], pos[j], is_k ? 0 : 1, head);
      if (pok[j] && ok_pos) reinterpret_cast<bf16*>(a.kv.pool)[off + hi] = from_f<bf16>(y);
      else if (hi == 0 && is_k) raise_status(a.status, ST_POS_OVERFLOW);
    }
  }
}

// g * x rows for the next GEMM (hi/lo) and the tile's sums of squares of x.
__device__ __forceinline__ void next_input(const EpiArgs& a, int nt, int m0, int nrows, float g,
                                           const float (&xv)[EPI_RG]) {
  __shared__ float red[TC_BM / 32][EPI_RG];
  const int i = threadIdx.x, n = nt * TC_BM + i;
  bf16* lo = a.lo_off ? a.xn + (size_t)a.lo_off * a.ld_xn : nullptr;
  float sq[EPI_RG];
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) {
    sq[j] = xv[j] * xv[j];
    if (j < nrows) store_split<bf16>(a.xn, lo, (size_t)(m0 + j) * a.ld_xn + n, g * xv[j]);
  }
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) sq[j] = warp_sum(sq[j]);
  if ((i & 31) == 0)
#pragma unroll
    for (int j = 0; j < EPI_RG; ++j) red[i >> 5][j] = sq[j];
  __syncthreads();
  if (i < nrows) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < TC_BM / 32; ++w) t += red[w][i];
    a.ss_out[(size_t)(m0 + i) * (a.d / TC_BM) + nt] = t;
  }
}

// ---------------------------------------------------------------------------
// o / down (and, with prep = 1, the layer-0 input): grid (d / 128,
// ceil(M / EPI_RG)), 128 threads.  x += y; then the next GEMM's input.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(TC_BM) epi_resid_kernel(const EpiArgs a) {
  constexpr int C = 6;
  __shared__ __align__(16) float sU[EPI_RG * EPI_R];
  pdl_trigger();
  pdl_wait();
  const int nt = blockIdx.x;
  int m0, nrows;
  if (!row_group(a, &m0, &nrows)) return;
  const int i = threadIdx.x;
  const int n = nt * TC_BM + i;

  // ---- every global load first
  float xv[EPI_RG];
#pragma unroll
  for (int j = 0; j < EPI_RG; ++j) xv[j] = j < nrows ? a.x[(size_t)(m0 + j) * a.d + n] : 0.f;
  const float g = a.g_next ? to_f(a.g_next[n]) : 0.f;
  if (!a.prep) {
    PartLoad<C> LU, LP;
    BRow B;
    float gate[EPI_RG];
    if (a.lora) {
      u_issue(a, 0, m0, nrows, i, LU);
      brow_issue(a, 0, n, B);
      gate_issue(a, m0, nrows, gate);
    }
    part_issue(a.pv, nt, m0, nrows, i, LP);
    // ---- then the arithmetic
    float acc[EPI_RG];
    if (a.lora) {
      u_store(LU, nrows, i, sU);
      __syncthreads();
    }
    part_add(LP, nrows, acc);
    if (a.lora) lora_dot(B, sU, gate, acc);
#pragma unroll
    for (int j = 0; j < EPI_RG; ++j) {
      xv[j] += acc[j];
      if (j < nrows) a.x[(size_t)(m0 + j) * a.d + n] = xv[j];
    }
  }
  if (a.g_next) next_input(a, nt, m0, nrows, g, xv);
}

// ---------------------------------------------------------------------------
// gate|up -> silu(gate) * up: grid (F / 128, ceil(M / EPI_RG)), 256 threads:
// threads 0..127 take the gate tile, 128..255 the up tile of the same
// features, so each thread holds one tile's loads.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(2 * TC_BM) epi_swiglu_kernel(const EpiArgs a) {
  constexpr int C = 4;
  __shared__ float s_inv[EPI_RG];
  __shared__ float s_ss[EPI_RG * EPI_MAX_SS];
  __shared__ __align__(16) float sU[2][EPI_RG * EPI_R];
  __shared__ float sUp[EPI_RG][TC_BM];
  pdl_trigger();
  pdl_wait();
  const int ft = blockIdx.x;
  int m0, nrows;
  if (!row_group(a, &m0, &nrows)) return;
  const int half = threadIdx.x / TC_BM;      // 0: gate, 1: up
  const int i = threadIdx.x % TC_BM;
  const int f = ft * TC_BM + i;
  const int tile = half ? a.F / TC_BM + ft : ft;

  // ---- every global load first
  float ssv[4];
  ss_issue(a, m0, nrows, ssv);
  PartLoad<C> LP, LU;
  BRow B;
  float gate[EPI_RG];
  part_issue(a.pv, tile, m0, nrows, i, LP);
  if (a.lora) {
    u_issue(a, half, m0, nrows, i, LU);
    brow_issue(a, half, f, B);
    gate_issue(a, m0, nrows, gate);
  }
  // ---- then the arithmetic
  if (a.lora) u_store(LU, nrows, i, sU[half]);
  ss_finish(a, nrows, ssv, s_ss, s_inv);     // syncs: sU complete too
  float v[EPI_RG];
  part_add(LP, nrows, v);
  if (a.lora) lora_dot(B, sU[half], gate, v);
  if (half) {
#pragma unroll
    for (int j = 0; j < EPI_RG; ++j) sUp[j][i] = v[j];
  }
  __syncthreads();
  if (!half) {
    bf16* lo = a.lo_off ? a.h + (size_t)a.lo_off * a.F : nullptr;
#pragma unroll
    for (int j = 0; j < EPI_RG; ++j) {
      if (j < nrows) {
        const float gv = v[j] * s_inv[j], uv = sUp[j][i] * s_inv[j];
        store_split<bf16>(a.h, lo, (size_t)(m0 + j) * a.F + f, gv / (1.0f + expf(-gv)) * uv);
      }
    }
  }
}

}  // namespace uno
