// Gated-LoRA linear layer, SIMT form (fp32 models, and any shape the tensor-
// core kernel does not take).
//
//   Y[m, n] = sum_k X[m, k] W[n, k] + sum_j U[m, uoff + j] Bl[n, j]
//
// where U = gate(m) * (alpha / r) * X A^T was produced by a previous call of
// the same kernel with A as the weight and the EPI_GATED epilogue.  Output
// columns are split into segments (e.g. q | k | v) that each have their own
// weight, LoRA-B matrix and U column offset, so fused projections need no
// concatenated weight copy.  One warp computes NC output columns for MT rows;
// lanes stride over K with 16-byte loads and the partial sums are reduced
// with shuffles at the end.
#pragma once

#include "common.cuh"

namespace uno {

enum Epilogue : int {
  EPI_STORE = 0,      // out (model dtype) = acc * alpha
  EPI_STORE_F32 = 1,  // out (fp32) = acc * alpha
  EPI_ADD_F32 = 2,    // out (fp32) += acc            (residual stream)
  EPI_GATED = 3       // out (model dtype) = acc * alpha * row_gate[m]   (LoRA down-projection)
};

struct GemmSeg {
  const void* W;      // [n, K]
  const void* lB;     // [n, r] or null
  int n0, n;          // first output column, column count
  int u_off;          // column of U feeding this segment's LoRA-B
};

constexpr int GEMM_MAX_SEG = 6;

struct GemmParams {
  const void* X; int ldx;    // [M, K] model dtype
  int M, K, N;
  GemmSeg seg[GEMM_MAX_SEG]; int nseg;
  const void* U; int ldu; int r;   // LoRA-B extension (U null: none)
  int epi; void* out; int ldo; float alpha;
  const float* row_gate;
  int lo_off;        // > 0: X and U also hold lo rows (x - bf16(x)) this many rows below
  void* out_lo;      // EPI_GATED: where the lo part of the output goes (or null)
  // tensor-core DUMP launches: completion counter of the kernel that wrote X
  // and its CTA count (null: the launch waits with pdl_wait)
  const unsigned* dep; unsigned dep_count;
  unsigned long long dep_limit_ns;   // the counter wait gives up after this long
  // EPI_STORE_F32: element offset of each output row (null: row * ldo)
  const int64_t* out_row;
  unsigned* done;                    // tensor-core DUMP mode: completion counter (see TcParams)
};

template <typename T, int MT, int NC>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const GemmParams p) {
  constexpr int VEC = Vec16<T>::N;
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_base = (blockIdx.x * 8 + warp) * NC;
  const int m0 = blockIdx.y * MT;
  if (n_base >= p.N) return;
  const int mrows = min(MT, p.M - m0);

  const T* wrow[NC];
  const T* brow[NC];
  int uoff[NC];
  bool valid[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int n = n_base + c;
    valid[c] = n < p.N;
    int s = 0;
#pragma unroll
    for (int t = 1; t < GEMM_MAX_SEG; ++t)
      if (t < p.nseg && n >= p.seg[t].n0) s = t;
    const GemmSeg& g = p.seg[s];
    const int nn = valid[c] ? n - g.n0 : 0;
    wrow[c] = reinterpret_cast<const T*>(g.W) + (size_t)nn * p.K;
    brow[c] = g.lB ? reinterpret_cast<const T*>(g.lB) + (size_t)nn * p.r : nullptr;
    uoff[c] = g.u_off;
  }

  float acc[MT][NC];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[m][c] = 0.f;

  const T* X = reinterpret_cast<const T*>(p.X);
  for (int k = lane * VEC; k < p.K; k += 32 * VEC) {
    float w[NC][VEC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      if (valid[c]) Vec16<T>::load(wrow[c] + k, w[c]);
      else
#pragma unroll
        for (int e = 0; e < VEC; ++e) w[c][e] = 0.f;
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < mrows) {
        float xv[VEC];
        Vec16<T>::load(X + (size_t)(m0 + m) * p.ldx + k, xv);
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[m][c] = fmaf(w[c][e], xv[e], acc[m][c]);
      }
    }
  }
  if (p.U) {
    const T* U = reinterpret_cast<const T*>(p.U);
    for (int k = lane * VEC; k < p.r; k += 32 * VEC) {
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        if (!valid[c] || !brow[c]) continue;
        float w[VEC];
        Vec16<T>::load(brow[c] + k, w);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < mrows) {
            float xv[VEC];
            Vec16<T>::load(U + (size_t)(m0 + m) * p.ldu + uoff[c] + k, xv);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[m][c] = fmaf(w[e], xv[e], acc[m][c]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[m][c] = warp_sum(acc[m][c]);

  // lane (m*NC + c) % 32 writes element (m, c)
#pragma unroll
  for (int m = 0; m < MT; ++m) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      if (((m * NC + c) & 31) != lane || m >= mrows || !valid[c]) continue;
      const int row = m0 + m, n = n_base + c;
      const float v = acc[m][c];
      switch (p.epi) {
        case EPI_STORE:
          reinterpret_cast<T*>(p.out)[(size_t)row * p.ldo + n] = from_f<T>(v * p.alpha);
          break;
        case EPI_STORE_F32:
          reinterpret_cast<float*>(p.out)[(p.out_row ? (size_t)p.out_row[row] : (size_t)row * p.ldo) + n] =
              v * p.alpha;
          break;
        case EPI_ADD_F32:
          reinterpret_cast<float*>(p.out)[(size_t)row * p.ldo + n] += v;
          break;
        default: {
          const float y = v * p.alpha * p.row_gate[row];
          const T hi = from_f<T>(y);
          reinterpret_cast<T*>(p.out)[(size_t)row * p.ldo + n] = hi;
          if (p.out_lo) reinterpret_cast<T*>(p.out_lo)[(size_t)row * p.ldo + n] = from_f<T>(y - to_f(hi));
          break;
        }
      }
    }
  }
}

}  // namespace uno
