// libuno: host runtime and C ABI of the Psi-Spec decode iteration.
//
// One iteration per request (blog page "不砸掉重来，给自回归 LLM 装一对“扩散翅膀”：
// Uno 的无损加速之路", sections 一句话直觉 and Ψ-Spec 采样器：起草、验证、两种模式):
//   draft pass   rows [pending, MASK x B] at positions c..c+B, LoRA gated on
//                for the MASK rows -> logits (AR p_1 on row 0, q_i on row i)
//   draft_sample x_1 ~ p_1 (AR only), x_i ~ q_i for i = 2..B
//   verify pass  rows x_1..x_B at c+1..c+B, LoRA off -> p_2..p_{B+1}
//   spec_verify  accept prefix, residual redraw or bonus, commit
// Draft and verify share the paged KV cache: the draft pass writes the
// pending token's keys/values at position c (final) and scratch keys for the
// MASK rows at c+1..c+B, which the verify pass then overwrites.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include <map>
#include <mutex>
#include <tuple>

#include "../../include/uno.h"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "epilogue.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "gemm_tokm.cuh"
#include "layers.cuh"
#include "sampling.cuh"
#include "tree.cuh"

using namespace uno;

namespace {

// ---------------------------------------------------------------------------
// GEMM environment: tensor-core workspace and the TMA descriptor cache.
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

struct MapKey {
  const void* p;
  uint64_t rows, cols, ld;
  uint32_t box_rows;
  bool operator<(const MapKey& o) const {
    return std::tie(p, rows, cols, ld, box_rows) < std::tie(o.p, o.rows, o.cols, o.ld, o.box_rows);
  }
};

constexpr int TC_COUNTERS = 1 << 16;
// A completion-counter wait gives up (and raises the device flag) after this long.
constexpr unsigned long long DEP_WAIT_NS = 1000000000ull;
constexpr int TC_MIN_UNITS = 8;

// Process-wide launch counts per kernel path (read by uno_debug_launch_counts).
int64_t g_launches[4] = {0, 0, 0, 0};   // tc gemm, simt gemm, tc attention, simt attention

// cudaFuncSetAttribute acts on the current device only, so a kernel's
// dynamic shared-memory limit is raised once per device (`done` is the
// kernel's own per-device record; devices past its size are set every time).
constexpr int ATTR_DEVS = 64;
template <typename K>
cudaError_t smem_attr_once(K kernel, int bytes, bool* done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  if (dev >= 0 && dev < ATTR_DEVS && done[dev]) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < ATTR_DEVS) done[dev] = true;
  return e;
}

// The fused pass's small kernels prefer the largest shared-memory carveout:
// an SM running one of them then takes a GEMM or attention CTA (200+ KB)
// beside it without reconfiguring.
template <typename K>
void carveout_once(K kernel, bool* done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  if (dev >= 0 && dev < ATTR_DEVS && done[dev]) return;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                             (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && dev >= 0 && dev < ATTR_DEVS) done[dev] = true;
  else cudaGetLastError();   // a preference only: leave no error behind
}

// Launch with programmatic stream serialisation when `pdl`: the kernel may
// start while the previous kernel of the stream is still running; inside,
// pdl_wait() orders every access to data an earlier kernel wrote.
template <typename... KArgs, typename... Args>
void klaunch(bool pdl, cudaStream_t st, dim3 grid, dim3 block, size_t smem,
             void (*kernel)(KArgs...), Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaLaunchKernelEx(&cfg, kernel, args...);
}

// spec_verify's first stage.  Few (row, chunk) CTAs: the fused kernel (the
// last CTA of a row forms its lse, the last row decides; one launch).  Many:
// the reduction CTAs carry no counters and exit at once, and one CTA per
// request combines and decides (one launch more, HBM kept busy).
constexpr long long VERIFY_SPLIT_CTAS = 4096;
// Returns the number of kernels launched.
template <bool FILT>
int launch_verify_t(bool pdl, cudaStream_t st, const VerifyArgs& a, int n_req, long long split_ctas) {
  const dim3 grid(a.nch, n_req * a.rows_red);
  if ((long long)a.nch * n_req * a.rows_red <= split_ctas) {
    klaunch(pdl, st, grid, dim3(SAMPLE_THREADS), 0, spec_verify_kernel<FILT>, a);
    return 1;
  }
  klaunch(pdl, st, dim3((a.nch + 1) / 2, n_req * a.rows_red), dim3(SAMPLE_THREADS), 0,
          spec_reduce_kernel<FILT>, a);
  klaunch(pdl, st, dim3(n_req), dim3(SAMPLE_THREADS), 0, spec_decide_kernel<FILT>, a);
  return 2;
}
// FILT: the p and q rows carry nucleus filters (a.filt_p, a.filt_q).
int launch_verify(bool pdl, cudaStream_t st, const VerifyArgs& a, int n_req,
                  long long split_ctas = VERIFY_SPLIT_CTAS, bool filt = false) {
  return filt ? launch_verify_t<true>(pdl, st, a, n_req, split_ctas)
              : launch_verify_t<false>(pdl, st, a, n_req, split_ctas);
}
void launch_resid(bool pdl, cudaStream_t st, const VerifyArgs& a, int n_req, bool filt) {
  if (filt) klaunch(pdl, st, dim3(a.nch, n_req), dim3(SAMPLE_THREADS), 0, spec_resid_kernel<true>, a);
  else klaunch(pdl, st, dim3(a.nch, n_req), dim3(SAMPLE_THREADS), 0, spec_resid_kernel<false>, a);
}
void launch_sample(bool pdl, cudaStream_t st, dim3 grid, const SampleArgs& a) {
  if (a.filt) klaunch(pdl, st, grid, dim3(SAMPLE_THREADS), 0, sample_rows_kernel<true>, a);
  else klaunch(pdl, st, grid, dim3(SAMPLE_THREADS), 0, sample_rows_kernel<false>, a);
}
// The nucleus threshold of n_req * a.rows_per_req rows (false: the kernel's
// shared-memory size could not be set).
bool launch_top_p(bool pdl, cudaStream_t st, const TopPArgs& a, int n_req) {
  static bool attr[ATTR_DEVS] = {};
  if (smem_attr_once(top_p_kernel, NUC_SMEM, attr) != cudaSuccess) return false;
  klaunch(pdl, st, dim3(n_req * a.rows_per_req), dim3(NUC_THREADS), NUC_SMEM, top_p_kernel, a);
  return true;
}

struct GemmEnv {
  int sm_count = 148;
  int x_rows_alloc = 0;           // rows the activation buffers hold (>= any box)
  float* ws = nullptr;            // [sm_count][2][256][128] fp32 partial tiles
  float* part = nullptr;          // DUMP-mode part slots
  size_t part_bytes = 0;
  unsigned* counters = nullptr;   // [TC_COUNTERS], zero, left zero
  int32_t* status = nullptr;
  std::map<MapKey, CUtensorMap> maps;
  bool tc_disabled = false;
  bool pdl = false;               // launch with programmatic stream serialisation

  static size_t ws_bytes(int sm) { return (size_t)sm * 2 * 256 * TC_BM * 4; }

  // bf16 (or fp16) 2-D row-major tensor [rows, cols] with row stride ld
  // elements; box of 64 columns (128 bytes, 128-byte swizzle) by box_rows rows.
  const CUtensorMap* map(const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                         uint32_t box_rows, bool fp16 = false) {
    MapKey k{base, rows, cols, ld, box_rows | (fp16 ? 0x80000000u : 0u)};
    auto it = maps.find(k);
    if (it != maps.end()) return &it->second;
    EncodeTiledFn f = encode_fn();
    if (!f) return nullptr;
    CUtensorMap m;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)TC_BK, box_rows};
    const cuuint32_t es[2] = {1, 1};
    if (f(&m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
          const_cast<void*>(base), dims, strides, box, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return nullptr;
    return &maps.emplace(k, m).first->second;
  }
};

// Stream-K shape of a DUMP-mode launch (what its epilogue kernel needs).
struct DumpShape {
  int NT = 0, units = 0, grid = 0, KBt = 0, m_tiles = 0, n_tiles = 0;
};

// Token tile width by row count: with split (hi/lo) activations the MMA's N
// holds 2 NT columns, so NT <= 128 and larger passes take several m-tiles.
int tc_nt(int M, bool split) {
  return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : (M <= 128 || split) ? 128 : 256;
}

// Part slots a DUMP-mode GEMM of M rows and N columns writes, in bytes.
size_t dump_bytes(int M, int N, int sm_count, bool split) {
  const int NT = tc_nt(M, split);
  const size_t slots = (size_t)((N + TC_BM - 1) / TC_BM) * ((M + NT - 1) / NT) + sm_count;
  return slots * NT * TC_BM * 4;
}

template <int NT, bool SPLIT, bool DUMP, int KPS>
bool launch_tc(GemmEnv& env, const GemmParams& p, cudaStream_t st, DumpShape* shape = nullptr) {
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  // A box may not be larger than the tensor: the activation tensors are
  // described with at least NT rows (the buffers hold x_rows_alloc >= 256
  // rows); rows past M only feed output columns the epilogue never stores.
  // In split mode they also cover the lo rows lo_off below.
  const uint64_t xrows = (SPLIT ? (uint64_t)p.lo_off : 0) + std::max<uint64_t>(p.M, NT);
  if ((uint64_t)env.x_rows_alloc < xrows) return false;
  for (int s = 0; s < p.nseg; ++s)
    if (p.seg[s].n < TC_BM) return false;
  if (p.U && p.nseg > 3) return false;   // LoRA-B maps: three segments
  const CUtensorMap* mx = env.map(p.X, xrows, p.K, p.ldx, NT);
  if (!mx) return false;
  maps.x = *mx;
  maps.u = *mx;
  if (p.U) {
    const CUtensorMap* mu = env.map(p.U, xrows, p.ldu, p.ldu, NT);
    if (!mu) return false;
    maps.u = *mu;
  }
  TcParams tp{};
  tp.M = p.M;
  tp.N = p.N;
  tp.KB = p.K / (TC_BK * KPS);
  tp.RB = p.U ? p.r / (TC_BK * KPS) : 0;
  tp.nseg = p.nseg;
  for (int s = 0; s < p.nseg; ++s) {
    const GemmSeg& g = p.seg[s];
    const CUtensorMap* mw = env.map(g.W, g.n, p.K, p.K, TC_BM);
    if (!mw) return false;
    maps.w[s] = *mw;
    if (s < 3) maps.b[s] = *mw;
    if (p.U) {
      if (!g.lB) return false;
      const CUtensorMap* mb = env.map(g.lB, g.n, p.r, p.r, TC_BM);
      if (!mb) return false;
      maps.b[s] = *mb;
    }
    tp.seg[s] = TcSeg{g.n0, g.n, g.u_off};
  }
  tp.n_tiles = (p.N + TC_BM - 1) / TC_BM;
  tp.m_tiles = (p.M + NT - 1) / NT;
  if ((long long)tp.n_tiles * tp.m_tiles > TC_COUNTERS) return false;
  // the device's stream-K arithmetic is 32-bit: units * grid < 2^32
  if ((long long)tp.n_tiles * tp.m_tiles * (tp.KB + tp.RB) * env.sm_count >= (1LL << 32)) return false;
  tp.units = tp.n_tiles * tp.m_tiles * (tp.KB + tp.RB);
  // at least TC_MIN_UNITS k-blocks per CTA: a tile is then cut into few
  // parts and its last contributor has few partials to add
  tp.grid = std::max(1, std::min(env.sm_count, tp.units / TC_MIN_UNITS));
  // several token m-tiles (max batch, prefill chunks): groups of m_tiles CTAs
  // that read each weight k-block together (measured at M = 1360 without
  // them: every CTA re-read its weight tile from HBM once per m-tile, 11x
  // the weight bytes)
  tp.mgroups = 0;
  if (!DUMP && tp.m_tiles >= 2) {
    const int g = std::min(env.sm_count / tp.m_tiles, tp.n_tiles * (tp.KB + tp.RB) / TC_MIN_UNITS);
    if (g >= 1) {
      tp.mgroups = g;
      tp.grid = g * tp.m_tiles;
    }
  }
  tp.max_parts = 2;
  tp.epi = p.epi;
  tp.out = p.out;
  tp.ldo = p.ldo;
  tp.alpha = p.alpha;
  tp.row_gate = p.row_gate;
  tp.ws = env.ws;
  tp.counters = env.counters;
  if (DUMP) {
    if (!env.part || dump_bytes(p.M, p.N, env.sm_count, SPLIT) > env.part_bytes) return false;
    tp.ws = env.part;
    if (shape) *shape = DumpShape{NT, tp.units, tp.grid, tp.KB + tp.RB, tp.m_tiles, tp.n_tiles};
  }
  tp.status = env.status;
  tp.lo_off = SPLIT ? p.lo_off : 0;
  tp.out_lo = p.out_lo;
  tp.dep = DUMP ? p.dep : nullptr;
  tp.dep_count = p.dep_count;
  tp.dep_limit_ns = p.dep_limit_ns ? p.dep_limit_ns : DEP_WAIT_NS;
  tp.out_row = p.out_row;
  tp.done = DUMP ? p.done : nullptr;

  using Cfg = TcCfg<NT, SPLIT, KPS>;
  static bool attr[ATTR_DEVS] = {};
  if (smem_attr_once(gemm_tc_kernel<NT, SPLIT, DUMP, KPS>, Cfg::SMEM, attr) != cudaSuccess)
    return false;
  klaunch(env.pdl, st, dim3(tp.grid), dim3(TC_THREADS), Cfg::SMEM,
          gemm_tc_kernel<NT, SPLIT, DUMP, KPS>, maps, tp);
  g_launches[0]++;
  return true;
}

// The tokens-in-M form (gemm_tokm.cuh) for split inputs of more than one
// token tile, not DUMP, fp32 outputs (stored or added: every projection of
// the unfused pass; the LoRA-A products keep the other form): every segment
// but the last a whole number of 256-row weight tiles, 16-byte aligned output
// rows, no row map.  False: not taken, nothing launched.
bool launch_tokm(GemmEnv& env, const GemmParams& p, cudaStream_t st) {
  if (p.lo_off <= 0 || p.M <= TK_BM || p.out_row) return false;
  if (p.epi != EPI_STORE_F32 && p.epi != EPI_ADD_F32) return false;
  for (int s = 0; s + 1 < p.nseg; ++s)
    if (p.seg[s].n % TK_BN) return false;
  if (p.ldo % 4 || ((uintptr_t)p.out & 15)) return false;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  const uint64_t xrows = (uint64_t)p.lo_off + std::max<uint64_t>(p.M, TK_BM);
  if ((uint64_t)env.x_rows_alloc < xrows) return false;
  for (int s = 0; s < p.nseg; ++s)
    if (p.seg[s].n < TC_BM) return false;
  if (p.U && p.nseg > 3) return false;   // LoRA-B maps: three segments
  const CUtensorMap* mx = env.map(p.X, xrows, p.K, p.ldx, TK_BM);
  if (!mx) return false;
  maps.x = *mx;
  maps.u = *mx;
  if (p.U) {
    const CUtensorMap* mu = env.map(p.U, xrows, p.ldu, p.ldu, TK_BM);
    if (!mu) return false;
    maps.u = *mu;
  }
  TcParams tp{};
  tp.M = p.M;
  tp.N = p.N;
  tp.KB = p.K / TC_BK;
  tp.RB = p.U ? p.r / TC_BK : 0;
  tp.nseg = p.nseg;
  for (int s = 0; s < p.nseg; ++s) {
    const GemmSeg& g = p.seg[s];
    const CUtensorMap* mw = env.map(g.W, g.n, p.K, p.K, TC_BM);
    if (!mw) return false;
    maps.w[s] = *mw;
    if (s < 3) maps.b[s] = *mw;
    if (p.U) {
      if (!g.lB) return false;
      const CUtensorMap* mb = env.map(g.lB, g.n, p.r, p.r, TC_BM);
      if (!mb) return false;
      maps.b[s] = *mb;
    }
    tp.seg[s] = TcSeg{g.n0, g.n, g.u_off};
  }
  tp.n_tiles = (p.N + TK_BN - 1) / TK_BN;
  tp.m_tiles = (p.M + TK_BM - 1) / TK_BM;
  if ((long long)tp.n_tiles * tp.m_tiles > TC_COUNTERS) return false;
  if ((long long)tp.n_tiles * tp.m_tiles * (tp.KB + tp.RB) * env.sm_count >= (1LL << 32)) return false;
  tp.units = tp.n_tiles * tp.m_tiles * (tp.KB + tp.RB);
  tp.grid = std::max(1, std::min(env.sm_count, tp.units / TC_MIN_UNITS));
  tp.mgroups = 0;
  const int g = std::min(env.sm_count / tp.m_tiles, tp.n_tiles * (tp.KB + tp.RB) / TC_MIN_UNITS);
  if (g >= 1) {
    tp.mgroups = g;
    tp.grid = g * tp.m_tiles;
  }
  tp.max_parts = 2;
  tp.epi = p.epi;
  tp.out = p.out;
  tp.ldo = p.ldo;
  tp.alpha = p.alpha;
  tp.row_gate = p.row_gate;
  tp.ws = env.ws;
  tp.counters = env.counters;
  tp.status = env.status;
  tp.lo_off = p.lo_off;
  tp.out_lo = p.out_lo;
  tp.dep_limit_ns = DEP_WAIT_NS;
  static bool attr[ATTR_DEVS] = {};
  if (smem_attr_once(gemm_tokm_kernel, TkCfg::SMEM, attr) != cudaSuccess) return false;
  klaunch(env.pdl, st, dim3(tp.grid), dim3(TC_THREADS), TkCfg::SMEM, gemm_tokm_kernel, maps, tp);
  g_launches[0]++;
  return true;
}

// Whether the tensor-core kernel takes this bf16 GEMM: K and r in 64-element
// blocks, every segment but the last a whole number of 128-row tiles, 16-byte
// aligned rows.
bool tc_shape_ok(const GemmParams& p) {
  if (p.K % TC_BK || (p.U && p.r % TC_BK) || p.ldx % 8 || (p.U && p.ldu % 8)) return false;
  for (int s = 0; s + 1 < p.nseg; ++s)
    if (p.seg[s].n % TC_BM) return false;
  for (int s = 0; s < p.nseg; ++s)
    if ((uintptr_t)p.seg[s].W & 15 || (p.U && ((uintptr_t)p.seg[s].lB & 15))) return false;
  return ((uintptr_t)p.X & 15) == 0 && (!p.U || ((uintptr_t)p.U & 15) == 0);
}

template <typename T>
void gemm_simt_dispatch(const GemmParams& p, cudaStream_t st, bool pdl) {
  const dim3 block(256);
  g_launches[1]++;
  if (p.M <= 8) {
    klaunch(pdl, st, dim3((p.N + 31) / 32, (p.M + 7) / 8), block, 0, gemm_simt_kernel<T, 8, 4>, p);
  } else if (p.M <= 16) {
    klaunch(pdl, st, dim3((p.N + 31) / 32, (p.M + 15) / 16), block, 0, gemm_simt_kernel<T, 16, 4>, p);
  } else {
    klaunch(pdl, st, dim3((p.N + 15) / 16, (p.M + 31) / 32), block, 0, gemm_simt_kernel<T, 32, 2>, p);
  }
}

// Tile width NT by row count; hi/lo split activations up to 128 rows.
template <bool DUMP, int KPS>
bool launch_tc_kps(GemmEnv& env, const GemmParams& p, cudaStream_t st, DumpShape* shape) {
  if (p.lo_off > 0) {
    if (p.M <= 16) return launch_tc<16, true, DUMP, KPS>(env, p, st, shape);
    if (p.M <= 32) return launch_tc<32, true, DUMP, KPS>(env, p, st, shape);
    if (p.M <= 64) return launch_tc<64, true, DUMP, KPS>(env, p, st, shape);
    return launch_tc<128, true, DUMP, KPS>(env, p, st, shape);
  }
  if (p.M <= 16) return launch_tc<16, false, DUMP, KPS>(env, p, st, shape);
  if (p.M <= 32) return launch_tc<32, false, DUMP, KPS>(env, p, st, shape);
  if (p.M <= 64) return launch_tc<64, false, DUMP, KPS>(env, p, st, shape);
  if (p.M <= 128) return launch_tc<128, false, DUMP, KPS>(env, p, st, shape);
  return launch_tc<256, false, DUMP, KPS>(env, p, st, shape);
}
// Two k-blocks per stage where K and the adapter rank allow it.
template <bool DUMP>
bool launch_tc_any(GemmEnv& env, const GemmParams& p, cudaStream_t st, DumpShape* shape) {
  if (p.K % (2 * TC_BK) == 0 && (!p.U || p.r % (2 * TC_BK) == 0))
    return launch_tc_kps<DUMP, 2>(env, p, st, shape);
  return launch_tc_kps<DUMP, 1>(env, p, st, shape);
}

// Runs one gated-LoRA GEMM: tcgen05 for bf16 shapes it takes, SIMT otherwise.
template <typename T>
void gemm_run(GemmEnv& env, const GemmParams& p, cudaStream_t st) {
  if (p.M <= 0 || p.N <= 0) return;
  if (sizeof(T) == 2 && !env.tc_disabled && tc_shape_ok(p) &&
      (launch_tokm(env, p, st) || launch_tc_any<false>(env, p, st, nullptr)))
    return;
  gemm_simt_dispatch<T>(p, st, env.pdl);
}

// DUMP-mode launch of a bf16 GEMM (false: the tensor-core kernel cannot take
// it, nothing was launched).
bool gemm_run_dump(GemmEnv& env, const GemmParams& p, cudaStream_t st, DumpShape* shape) {
  if (p.M <= 0 || p.N <= 0 || env.tc_disabled || !tc_shape_ok(p)) return false;
  return launch_tc_any<true>(env, p, st, shape);
}

}  // namespace

struct uno_ctx {
  uno_shape s{};
  int r = 0, B = 0, max_batch = 0, max_ctx = 0;
  float alpha = 0.f, lscale = 0.f;
  uint64_t seed = 0;
  cudaStream_t stream = nullptr;
  size_t esz = 4;  // element size of the model dtype

  // weights (borrowed)
  const void *embed = nullptr, *lm_head = nullptr, *final_norm = nullptr;
  std::vector<const void*> attn_norm, ffn_norm;
  std::vector<const void*> w[UNO_N_PROJ], lA[UNO_N_PROJ], lB[UNO_N_PROJ];

  // KV pool and request slots
  KvLayout kv{};
  void* kv_pool = nullptr;
  int32_t* d_page_table = nullptr;
  int32_t *d_cached = nullptr, *d_pending = nullptr;
  uint32_t* d_stream = nullptr;
  std::vector<int> free_pages;
  std::vector<int> slot_used;
  std::vector<int32_t> h_page_table;

  // activations (sized for M_max rows)
  int M_max = 0;
  float* x = nullptr;          // [M, d] fp32 residual
  void* xn = nullptr;          // [M, max(d, F)] GEMM input (normed rows, SwiGLU output)
  float* qkv = nullptr;        // [M, (H + 2 Hkv) hd] fp32 projection output
  void* qbuf = nullptr;        // [M, H hd] rotated q (attention input)
  void* attn = nullptr;        // [M, H hd]
  float* gu = nullptr;         // [M, 2F] fp32 gate|up output
  void* U = nullptr;           // [M, 3r] LoRA intermediate
  float* ss = nullptr;         // [M, d / 128] sums of squares of x per 128-column tile
  bool fused = false;          // the fused bf16 layer pipeline applies to this model
  bool fused_enabled = true;
  int verify_split_ctas = 4096;   // spec_verify: split form above this many CTAs
  int32_t *row_pos = nullptr, *row_slot = nullptr;
  float* row_gate = nullptr;
  int32_t *row_cslot = nullptr, *row_blk = nullptr;   // training form: per-row key ranges
  int32_t* train_slots = nullptr;                     // [2 max_batch] slots of a training pass
  // cohort step (allocated by its first call)
  float* coh_logits = nullptr;     // [2 max_batch (B+1), V]: per-slot draft rows, then verify rows
  int32_t* coh_drafts = nullptr;   // [max_batch, B] drafted block per slot
  float* coh_lse_q = nullptr;      // [max_batch, B]
  int32_t* coh_phase = nullptr;    // [max_batch] 0: to be drafted, 1: drafted
  int32_t* coh_rows = nullptr;     // [max_batch] slots of the pass: drafting cohort, then verifying
  int64_t* coh_rowoff = nullptr;   // [M_max] logits offset of each row
  int coh_n_draft = 0;
  // tree sampler (tree_k >= 2; set by uno_set_tree)
  int tree_k = 1;
  float* logits_t = nullptr;       // [max_batch, k, B, V] chain verify logits
  float* lse_t = nullptr;          // [max_batch, k, B]
  int32_t* tree_chains = nullptr;  // [max_batch, k, B]
  float* tree_resid = nullptr;     // [max_batch, 2, V]
  int32_t* tree_walk = nullptr;    // [max_batch, 3]
  int32_t* tree_pages = nullptr;   // [max_batch, TREE_MAX_K, 2]
  std::vector<int32_t> h_tree_pages;   // reserved scratch pages (host copy)
  size_t tree_cap_k = 0;           // chains the buffers are sized for
  RowKeys keys{};                                     // key ranges of the current pass
  // completion counters of the fused pass (GEMMs wait on the kernel before
  // them through these instead of pdl_wait), zeroed by each pass's first kernel
  unsigned* dep_ctr = nullptr;
  int n_dep_ctr = 0;
  bool counter_sync = true;
  unsigned long long dep_limit_ns = DEP_WAIT_NS;   // test tap: counter-wait limit
  unsigned dep_extra = 0;                          // test tap: added to every counter target
  int fixed_accept = -1;                           // bench tap: forced a (first token + accepted)
  float *cos_t = nullptr, *sin_t = nullptr;
  int max_pos = 0;

  // logits and sampler state
  float *logits_d = nullptr, *logits_v = nullptr;   // [max_batch, B+1, V], [max_batch, B, V]
  int32_t* drafts = nullptr;                        // [max_batch, B]
  float* lse_q = nullptr;                           // [max_batch, B]
  int nch = 1, ch = 1;
  float2* partial = nullptr;                        // [max_batch * 2B, nch]
  float* lse_ws = nullptr;                          // [max_batch * 2B]
  unsigned* row_counter = nullptr;                  // [max_batch * 2B]
  unsigned* req_counter = nullptr;                  // [max_batch]
  int32_t* at_ws = nullptr;                         // [max_batch]
  float top_p = 1.f;                                // nucleus filter (1: off)
  RowFilter* filt_d = nullptr;                      // [max_batch, B+1] nucleus of draft rows
  RowFilter* filt_v = nullptr;                      // [max_batch, B]   nucleus of verify rows
  float* resid_part = nullptr;                      // [max_batch, nch]
  unsigned* resid_counter = nullptr;                // [max_batch]

  // attention split workspace
  float* att_ws = nullptr;
  size_t att_ws_floats = 0;
  unsigned* att_counters = nullptr;
  int att_groups_max = 0;

  int32_t* d_status = nullptr;
  int last_n_req = 0;
  std::string err;
  GemmEnv genv;
  CUtensorMap kv_map;            // the pool as a 2-D fp16 [rows, head_dim] tensor
  CUtensorMap q_map;             // q rows as a 3-D fp16 [2 M_max rows, H, head_dim] tensor
  bool kv_map_ok = false;

  // CUDA graphs of whole steps, keyed by their arguments
  struct GraphEntry {
    int kind, n_req;
    const void *a, *b, *c, *d;
    int seen = 0;
    cudaGraphExec_t exec = nullptr;
    int64_t launches[UNO_K_N] = {};
    double bytes[UNO_K_N] = {};
    int64_t glaunch[4] = {};
  };
  std::vector<GraphEntry> graphs;
  bool graphs_enabled = true;
  cudaStream_t cap_stream = nullptr;

  // profiling tap
  unsigned prof_mask = 0;
  int64_t prof_launches[UNO_K_N] = {};
  double prof_bytes[UNO_K_N] = {};
  struct ProfRec { int cls, m, n, k, r; cudaEvent_t a, b; };
  std::vector<ProfRec> prof_recs;
  std::vector<uno_prof_record> prof_done;   // records of the last uno_profile_end
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_next = 0;
};

namespace {
cudaEvent_t next_event(uno_ctx* c) {
  if (c->ev_next == c->ev_pool.size()) {
    cudaEvent_t e;
    cudaEventCreate(&e);
    c->ev_pool.push_back(e);
  }
  return c->ev_pool[c->ev_next++];
}

// Counts a launch of class `cls` and, when that class is profiled, brackets it
// with an event pair on the context stream.
struct Prof {
  uno_ctx* c;
  int cls;
  int m = 0, n = 0, k = 0, r = 0;
  cudaEvent_t a = nullptr, b = nullptr;
  Prof(uno_ctx* c_, int cls_, double bytes, int m_ = 0, int n_ = 0, int k_ = 0, int r_ = 0)
      : c(c_), cls(cls_), m(m_), n(n_), k(k_), r(r_) {
    c->prof_launches[cls]++;
    c->prof_bytes[cls] += bytes;
    if (c->prof_mask & (1u << cls)) {
      a = next_event(c);
      b = next_event(c);
      cudaEventRecord(a, c->stream);
    }
  }
  ~Prof() {
    if (b) {
      cudaEventRecord(b, c->stream);
      c->prof_recs.push_back({cls, m, n, k, r, a, b});
    }
  }
};
}  // namespace

namespace {

constexpr int PREFILL_CHUNK = 512;
constexpr int FUSED_MAX_ROWS = 128;   // rows of a pass the fused pipeline takes
// Largest vocabulary: 64 chunks of 8192 logits (one thread combines a row's
// chunk pairs serially).
constexpr int MAX_VOCAB = 64 * 8192;

int fail(uno_ctx* c, int code, const std::string& msg) {
  if (c) c->err = msg;
  return code;
}

#define CK(call)                                                                            \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess)                                                                  \
      return fail(c, UNO_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_));     \
  } while (0)

template <typename P>
cudaError_t dalloc(P** p, size_t bytes) {
  return cudaMalloc((void**)p, bytes ? bytes : 16);
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// ---------------------------------------------------------------------------
// GEMM dispatch.
// ---------------------------------------------------------------------------
struct Gemm {
  GemmParams p{};
  Gemm(const void* X, int ldx, int M, int K) {
    p.X = X; p.ldx = ldx; p.M = M; p.K = K; p.N = 0; p.nseg = 0; p.U = nullptr; p.r = 0;
    p.alpha = 1.f; p.row_gate = nullptr;
  }
  Gemm& seg(const void* W, int n, const void* lB = nullptr, int u_off = 0) {
    p.seg[p.nseg] = GemmSeg{W, lB, p.N, n, u_off};
    p.nseg++;
    p.N += n;
    return *this;
  }
  Gemm& lora(const void* U, int ldu, int r) { p.U = U; p.ldu = ldu; p.r = r; return *this; }
  Gemm& epi(int e, void* out, int ldo, float alpha = 1.f, const float* gate = nullptr) {
    p.epi = e; p.out = out; p.ldo = ldo; p.alpha = alpha; p.row_gate = gate;
    return *this;
  }
};

// Algorithmic bytes of one GEMM launch: weights, LoRA-B, activations and U
// read once, outputs written once (read too for the residual add).
double gemm_bytes(const GemmParams& p, size_t esz) {
  double b = (double)esz * ((double)p.N * p.K + (double)p.M * p.K);
  if (p.U) b += (double)esz * ((double)p.N * p.r + (double)p.M * p.r);
  const double out = (double)p.M * p.N;
  if (p.epi == EPI_STORE || p.epi == EPI_GATED) b += out * esz;
  else if (p.epi == EPI_STORE_F32) b += out * 4;
  else b += out * 8;
  return b;
}

template <typename T>
void launch_gemm(uno_ctx* c, const Gemm& g, cudaStream_t st) {
  const GemmParams& p = g.p;
  if (p.M <= 0 || p.N <= 0) return;
  Prof prof(c, UNO_K_GEMM, gemm_bytes(p, sizeof(T)), p.M, p.N, p.K, p.U ? p.r : 0);
  gemm_run<T>(c->genv, p, st);
}

// ---------------------------------------------------------------------------
// Attention dispatch.
// ---------------------------------------------------------------------------
template <typename T, int HD>
int launch_attn_hd(uno_ctx* c, AttnParams& p, int n_req, cudaStream_t st) {
  const size_t smem = (size_t)(ATT_MAXQ * HD + ATT_KT * (HD + 1) + ATT_KT * HD) * sizeof(float);
  static bool attr[ATTR_DEVS] = {};
  CK(smem_attr_once(attn_simt_kernel<T, HD>, (int)smem, attr));
  const dim3 grid(p.n_splits, p.n_qtiles, n_req * p.Hkv);
  Prof prof(c, UNO_K_ATTN, 0.0);
  klaunch(c->genv.pdl, st, grid, dim3(ATT_THREADS), smem, attn_simt_kernel<T, HD>, p);
  g_launches[3]++;
  return UNO_OK;
}

// Completion counters around the tensor-core attention of the fused pass:
// the q|k|v epilogue's (dep, its CTA count) and one the attention CTAs add
// to, which the split merge waits on.
struct AttnSync {
  const unsigned* dep = nullptr;
  unsigned dep_n = 0;
  unsigned* done = nullptr;
};

template <int HD>
int launch_attn_tc(uno_ctx* c, int layer, int n_req, int rows_per_req, bool decode,
                   void* out_lo, const void* l2_pf, size_t l2_pf_bytes, const AttnSync& sync) {
  const uno_shape& s = c->s;
  AttnTcParams p{};
  p.q = (const f16*)c->qbuf;
  p.q_lo_row = c->M_max;
  p.ld_q = s.n_heads * HD;
  p.out = (bf16*)c->attn;
  p.ld_out = s.n_heads * HD;
  p.out_lo = (bf16*)out_lo;
  p.layer = layer;
  p.H = s.n_heads;
  p.Hkv = s.n_kv_heads;
  p.n_pages = c->kv.n_pages;
  p.pages_per_req = c->kv.pages_per_req;
  p.page_table = c->d_page_table;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  p.rows_per_req = rows_per_req;
  p.row_pos = c->row_pos;
  p.row_slot = c->row_slot;
  p.keys = c->keys;
  const int G = s.n_heads / s.n_kv_heads;
  p.n_qtiles = ceil_div(rows_per_req, ATC_QROWS / G);
  const int groups = n_req * s.n_kv_heads * p.n_qtiles;
  int S = 1;
  const int sm = c->genv.sm_count;
  if (decode && groups < sm) {
    // one CTA per SM (shared memory): at most sm_count CTAs, else a second wave
    S = sm / groups;
    S = std::max(1, std::min(std::min(S, c->kv.pages_per_req / 2), ATC_MAX_SPLITS));
  }
  // With more groups than SMs the attention runs unsplit, in several waves:
  // splitting to fill the last wave was measured slower at 80 requests (three
  // splits: 611 us of attention plus 137 us of merge per layer-pass against
  // 640 us unsplit)
  while (S > 1 && (size_t)groups * S * ATC_QROWS * atc_ws_row(HD) > c->att_ws_floats) --S;
  if (groups > c->att_groups_max) S = 1;
  p.n_splits = S;
  p.ws = c->att_ws;
  p.status = c->d_status;
  const bool pf_ok = l2_pf && l2_pf_bytes >= 16 && ((uintptr_t)l2_pf & 15) == 0;
  p.l2_pf = pf_ok ? (const char*)l2_pf : nullptr;
  p.l2_pf_bytes = pf_ok ? (unsigned long long)(l2_pf_bytes & ~(size_t)15) : 0ull;
  p.dep = sync.dep;
  p.dep_count = sync.dep ? sync.dep_n + c->dep_extra : 0u;
  p.dep_limit_ns = c->dep_limit_ns;
  p.done = S > 1 ? sync.done : nullptr;
  static bool attr[ATTR_DEVS] = {};
  CK(smem_attr_once(attn_tc_kernel<HD>, AtcCfg<HD>::SMEM, attr));
  {
    Prof prof(c, UNO_K_ATTN, 0.0);
    klaunch(c->genv.pdl, c->stream, dim3(S, p.n_qtiles, n_req * s.n_kv_heads), dim3(ATC_THREADS),
            AtcCfg<HD>::SMEM, attn_tc_kernel<HD>, c->kv_map, c->q_map, p);
  }
  g_launches[2]++;
  if (S > 1) {
    Prof prof(c, UNO_K_ATTN, 0.0);
    // only the rows a query tile can hold: tokens per request x heads per kv head
    const int rows = std::min(ATC_QROWS, rows_per_req * G);
    if (p.done) {
      p.dep = p.done;
      p.dep_count = (unsigned)(S * groups) + c->dep_extra;
      p.done = nullptr;
    }
    klaunch(c->genv.pdl, c->stream, dim3(ceil_div(rows, ATC_MERGE_ROWS), groups),
            dim3(HD, ATC_MERGE_ROWS), 0, attn_merge_kernel<HD>, p);
  }
  return UNO_OK;
}

// l2_pf (optional): weights of the next projection, prefetched into L2 by the
// tensor-core attention while it runs.
template <typename T>
int launch_attn(uno_ctx* c, int layer, int n_req, int rows_per_req, bool decode,
                void* out_lo, const void* l2_pf = nullptr, size_t l2_pf_bytes = 0,
                const AttnSync& sync = AttnSync{}) {
  const uno_shape& s = c->s;
  if (c->kv_map_ok) {
    if (s.head_dim == 128)
      return launch_attn_tc<128>(c, layer, n_req, rows_per_req, decode, out_lo, l2_pf, l2_pf_bytes,
                                 sync);
    if (s.head_dim == 64)
      return launch_attn_tc<64>(c, layer, n_req, rows_per_req, decode, out_lo, l2_pf, l2_pf_bytes,
                                sync);
  }
  // the SIMT attention waits on the grid dependency (sync unused)
  AttnParams p{};
  p.qkv = c->qbuf;
  p.q_lo = sizeof(T) == 2 ? (const char*)c->qbuf + (size_t)c->M_max * s.n_heads * s.head_dim * 2
                          : nullptr;
  p.ld_qkv = s.n_heads * s.head_dim;
  p.out = c->attn;
  p.ld_out = s.n_heads * s.head_dim;
  p.out_lo = out_lo;
  p.kv = c->kv;
  p.layer = layer;
  p.H = s.n_heads;
  p.Hkv = s.n_kv_heads;
  p.scale = 1.0f / sqrtf((float)s.head_dim);
  p.rows_per_req = rows_per_req;
  p.row_pos = c->row_pos;
  p.row_slot = c->row_slot;
  p.keys = c->keys;
  const int G = s.n_heads / s.n_kv_heads;
  const int TQ = ATT_MAXQ / G;
  p.n_qtiles = ceil_div(rows_per_req, TQ);
  const int groups = n_req * s.n_kv_heads * p.n_qtiles;
  int S = 1;
  if (decode) {
    S = ceil_div(2 * 148, groups);
    const int max_tiles = ceil_div(c->max_ctx + c->B + 2, ATT_KT);
    S = std::max(1, std::min(S, max_tiles / 8));
    while (S > 1 && (size_t)groups * S * ATT_MAXQ * (s.head_dim + 2) > c->att_ws_floats) --S;
    if (groups > c->att_groups_max) S = 1;
  }
  p.n_splits = S;
  p.ws = c->att_ws;
  p.counters = c->att_counters;
  switch (s.head_dim) {
    case 16: return launch_attn_hd<T, 16>(c, p, n_req, c->stream);
    case 32: return launch_attn_hd<T, 32>(c, p, n_req, c->stream);
    case 64: return launch_attn_hd<T, 64>(c, p, n_req, c->stream);
    case 128: return launch_attn_hd<T, 128>(c, p, n_req, c->stream);
    default: return fail(c, UNO_ERR_UNSUPPORTED, "head_dim must be 16, 32, 64 or 128");
  }
}

// ---------------------------------------------------------------------------
// One forward pass over M = n_req * rows_per_req rows.
// ---------------------------------------------------------------------------
template <typename T>
int forward(uno_ctx* c, int kind, int n_req, int rows_per_req, const int32_t* req_ids,
            const int32_t* prompt, int prefill_slot, int prefill_pos0, float* logits) {
  const uno_shape& s = c->s;
  const int M = n_req * rows_per_req;
  const int d = s.d_model, H = s.n_heads, Hkv = s.n_kv_heads, hd = s.head_dim, F = s.ffn_dim;
  const int r = c->r;
  const int qkv_ld = (H + 2 * Hkv) * hd;
  // the adapter is read by the passes with gated rows (draft, training form)
  const bool lora = (kind == PASS_DRAFT || kind == PASS_TRAIN || kind == PASS_COHORT);
  cudaStream_t st = c->stream;

  RowArgs ra{};
  ra.kind = kind;
  ra.rows_per_req = rows_per_req;
  ra.req_slot = req_ids;
  ra.cached = c->d_cached;
  ra.pending = c->d_pending;
  ra.drafts = c->drafts;
  ra.B = c->B;
  ra.prompt = prompt;
  ra.prefill_slot = prefill_slot;
  ra.mask_id = s.mask_id;
  ra.vocab = s.vocab;
  ra.max_batch = c->max_batch;
  ra.lora_scale = c->lscale;
  ra.row_pos = c->row_pos;
  ra.row_slot = c->row_slot;
  ra.row_gate = c->row_gate;
  ra.embed = c->embed;
  ra.d = d;
  ra.x = c->x;
  ra.status = c->d_status;
  ra.prefill_pos0 = prefill_pos0;
  ra.row_cslot = c->row_cslot;
  ra.row_blk = c->row_blk;
  ra.n_draft = c->coh_n_draft;
  ra.phase = c->coh_phase;
  ra.coh_drafts = c->coh_drafts;
  ra.row_off = c->coh_rowoff;
  ra.coh_v_row0 = (int64_t)c->max_batch * (c->B + 1);
  ra.tree_k = c->tree_k;
  ra.tree_chains = c->tree_chains;
  ra.tree_pages = c->tree_pages;
  ra.pt_rw = c->d_page_table;
  ra.pages_per_req = c->kv.pages_per_req;
  c->keys = (kind == PASS_TRAIN || kind == PASS_TREE) ? RowKeys{c->row_cslot, c->row_blk}
                                                     : RowKeys{nullptr, nullptr};
  {
    Prof prof(c, UNO_K_OTHER, 0.0);
    klaunch(c->genv.pdl, st, dim3(M), dim3(256), 0, build_rows_kernel<T>, ra);
  }
  auto other = [&](auto launch) {
    Prof prof(c, UNO_K_OTHER, 0.0);
    launch();
  };

  const int xn_ld = std::max(d, F);
  const int ldu = 3 * r;
  const int hhd = H * hd;
  // bf16 models feed every GEMM input as a hi/lo pair of bf16 rows
  // (x = hi + lo), the lo rows c->M_max rows below the hi rows.
  const bool split = sizeof(T) == 2;
  const int lo = split ? c->M_max : 0;
  auto lo_rows = [&](void* buf, int ld) -> T* {
    return split ? reinterpret_cast<T*>(buf) + (size_t)lo * ld : nullptr;
  };
  T* xn_lo = lo_rows(c->xn, xn_ld);
  T* act_lo = lo_rows(c->xn, F);
  T* attn_lo = lo_rows(c->attn, hhd);
  T* u_lo = lo_rows(c->U, ldu);
  auto gated = [&](Gemm& g) { g.epi(EPI_GATED, c->U, ldu, 1.f, c->row_gate); g.p.out_lo = u_lo; };
  for (int l = 0; l < s.n_layers; ++l) {
    other([&] {
      klaunch(c->genv.pdl, st, dim3(M), dim3(256), 0, rmsnorm_kernel<T, 256>, (const float*)c->x,
              (const T*)c->attn_norm[l], (T*)c->xn, xn_lo, d, xn_ld, s.rms_eps);
    });
    if (lora) {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->lA[UNO_PROJ_Q][l], r).seg(c->lA[UNO_PROJ_K][l], r).seg(c->lA[UNO_PROJ_V][l], r);
      gated(g);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->w[UNO_PROJ_Q][l], H * hd, lora ? c->lB[UNO_PROJ_Q][l] : nullptr, 0)
          .seg(c->w[UNO_PROJ_K][l], Hkv * hd, lora ? c->lB[UNO_PROJ_K][l] : nullptr, r)
          .seg(c->w[UNO_PROJ_V][l], Hkv * hd, lora ? c->lB[UNO_PROJ_V][l] : nullptr, 2 * r);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_STORE_F32, c->qkv, qkv_ld);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
    other([&] {
      klaunch(c->genv.pdl, st, dim3(M), dim3(256), 0, rope_kv_kernel<T>,
              (const float*)c->qkv,
              qkv_ld, (typename KvOf<T>::type*)c->qbuf,
              split ? (typename KvOf<T>::type*)c->qbuf + (size_t)c->M_max * hhd : nullptr, hhd,
              (const int32_t*)c->row_pos, (const int32_t*)c->row_slot,
              (const float*)c->cos_t, (const float*)c->sin_t, c->max_pos, H, Hkv, hd, c->kv, l,
              c->d_status);
    });
    {
      const int rc = launch_attn<T>(c, l, n_req, rows_per_req, kind != PASS_PREFILL, attn_lo);
      if (rc) return rc;
    }
    if (lora) {
      Gemm g(c->attn, hhd, M, hhd);
      g.seg(c->lA[UNO_PROJ_O][l], r);
      gated(g);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->attn, hhd, M, hhd);
      g.seg(c->w[UNO_PROJ_O][l], d, lora ? c->lB[UNO_PROJ_O][l] : nullptr, 0);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_ADD_F32, c->x, d);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
    other([&] {
      klaunch(c->genv.pdl, st, dim3(M), dim3(256), 0, rmsnorm_kernel<T, 256>, (const float*)c->x,
              (const T*)c->ffn_norm[l], (T*)c->xn, xn_lo, d, xn_ld, s.rms_eps);
    });
    if (lora) {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->lA[UNO_PROJ_GATE][l], r).seg(c->lA[UNO_PROJ_UP][l], r);
      gated(g);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->xn, xn_ld, M, d);
      g.seg(c->w[UNO_PROJ_GATE][l], F, lora ? c->lB[UNO_PROJ_GATE][l] : nullptr, 0)
          .seg(c->w[UNO_PROJ_UP][l], F, lora ? c->lB[UNO_PROJ_UP][l] : nullptr, r);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_STORE_F32, c->gu, 2 * F);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
    other([&] {
      klaunch(c->genv.pdl, st, dim3(M, ceil_div(F, 4 * 128)), dim3(128), 0, swiglu_kernel<T>,
              (const float*)c->gu, F,
              (T*)c->xn, act_lo);
    });
    if (lora) {
      Gemm g(c->xn, F, M, F);
      g.seg(c->lA[UNO_PROJ_DOWN][l], r);
      gated(g);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
    {
      Gemm g(c->xn, F, M, F);
      g.seg(c->w[UNO_PROJ_DOWN][l], d, lora ? c->lB[UNO_PROJ_DOWN][l] : nullptr, 0);
      if (lora) g.lora(c->U, ldu, r);
      g.epi(EPI_ADD_F32, c->x, d);
      g.p.lo_off = lo;
      launch_gemm<T>(c, g, st);
    }
  }
  if (logits) {
    other([&] {
      klaunch(c->genv.pdl, st, dim3(M), dim3(256), 0, rmsnorm_kernel<T, 256>, (const float*)c->x,
              (const T*)c->final_norm, (T*)c->xn, xn_lo, d, xn_ld, s.rms_eps);
    });
    Gemm g(c->xn, xn_ld, M, d);
    g.seg(c->lm_head, s.vocab).epi(EPI_STORE_F32, logits, s.vocab, 1.0f / s.temperature);
    g.p.lo_off = lo;
    g.p.out_row = kind == PASS_COHORT ? c->coh_rowoff : nullptr;
    launch_gemm<T>(c, g, st);
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

// ---------------------------------------------------------------------------
// One forward pass, bf16 models on the tensor cores: per layer four DUMP-mode
// weight streams, each followed by its fused epilogue (epilogue.cuh):
//
//   qkv GEMM [Wq|Wk|Wv (|Aq|Ak|Av)] -> epi_qkv   (LoRA-B, norm, RoPE, KV write)
//   attention (+ split merge)
//   o GEMM   [Wo (|Ao)]             -> epi_resid (LoRA-B, x +=, ffn-norm input)
//   gate|up  [Wg|Wu (|Ag|Au)]       -> epi_swiglu
//   down     [Wd (|Ad)]             -> epi_resid (LoRA-B, x +=, next attn-norm input)
//
// then the final RMSNorm and the LM head.  The LoRA A matrices ride in the
// same weight stream as W (draft pass only), so no pass ever launches a
// separate rank-r GEMM.
// ---------------------------------------------------------------------------
int forward_fused(uno_ctx* c, int kind, int n_req, int rows_per_req, const int32_t* req_ids,
                  const int32_t* prompt, int prefill_slot, int prefill_pos0, float* logits) {
  const uno_shape& s = c->s;
  const int M = n_req * rows_per_req;
  const int d = s.d_model, H = s.n_heads, Hkv = s.n_kv_heads, hd = s.head_dim, F = s.ffn_dim;
  const int r = c->r;
  const int qkv_n = (H + 2 * Hkv) * hd;
  const bool lora = (kind == PASS_DRAFT || kind == PASS_TRAIN || kind == PASS_COHORT) && r > 0;
  cudaStream_t st = c->stream;
  const bool pdl = c->genv.pdl;

  RowArgs ra{};
  ra.kind = kind;
  ra.rows_per_req = rows_per_req;
  ra.req_slot = req_ids;
  ra.cached = c->d_cached;
  ra.pending = c->d_pending;
  ra.drafts = c->drafts;
  ra.B = c->B;
  ra.prompt = prompt;
  ra.prefill_slot = prefill_slot;
  ra.mask_id = s.mask_id;
  ra.vocab = s.vocab;
  ra.max_batch = c->max_batch;
  ra.lora_scale = c->lscale;
  ra.row_pos = c->row_pos;
  ra.row_slot = c->row_slot;
  ra.row_gate = c->row_gate;
  ra.embed = c->embed;
  ra.d = d;
  ra.x = c->x;
  ra.status = c->d_status;
  ra.prefill_pos0 = prefill_pos0;
  // completion counters: each GEMM waits for the epilogue before it (its X
  // rows), each epilogue for its GEMM (the parts), the attention for the
  // q|k|v epilogue and the split merge for the attention, each through a
  // counter the producer's CTAs add to at their end; the o GEMM alone waits
  // on the grid dependency.  The counters are zeroed by build_rows.
  const bool csync = c->counter_sync && c->dep_ctr;
  int n_ctr = 0;
  const unsigned* dep = nullptr;   // counter of the last signalling kernel
  unsigned dep_n = 0;              // and its CTA count
  auto next_ctr = [&]() -> unsigned* {
    return (csync && n_ctr < c->n_dep_ctr) ? c->dep_ctr + n_ctr++ : nullptr;
  };
  ra.zero_ctr = csync ? c->dep_ctr : nullptr;
  ra.n_zero = c->n_dep_ctr;
  ra.row_cslot = c->row_cslot;
  ra.row_blk = c->row_blk;
  ra.n_draft = c->coh_n_draft;
  ra.phase = c->coh_phase;
  ra.coh_drafts = c->coh_drafts;
  ra.row_off = c->coh_rowoff;
  ra.coh_v_row0 = (int64_t)c->max_batch * (c->B + 1);
  ra.tree_k = c->tree_k;
  ra.tree_chains = c->tree_chains;
  ra.tree_pages = c->tree_pages;
  ra.pt_rw = c->d_page_table;
  ra.pages_per_req = c->kv.pages_per_req;
  c->keys = (kind == PASS_TRAIN || kind == PASS_TREE) ? RowKeys{c->row_cslot, c->row_blk}
                                                     : RowKeys{nullptr, nullptr};
  {
    Prof prof(c, UNO_K_OTHER, 0.0);
    klaunch(pdl, st, dim3(M), dim3(256), 0, build_rows_kernel<bf16>, ra);
  }

  const int xn_ld = std::max(d, F);
  const int hhd = H * hd;
  // every GEMM input is a hi/lo pair of bf16 rows (x = hi + lo), the lo rows
  // M_max rows below the hi rows
  const bool split = true;
  const int lo = c->M_max;
  bf16* attn_lo = (bf16*)c->attn + (size_t)lo * hhd;

  EpiArgs ea{};
  ea.M = M;
  ea.lo_off = lo;
  ea.n_ss = d / TC_BM;
  ea.d_model = (float)d;
  ea.eps = s.rms_eps;
  ea.q_out = (f16*)c->qbuf;
  ea.ld_q = hhd;
  ea.H = H; ea.Hkv = Hkv; ea.hd = hd;
  ea.row_pos = c->row_pos;
  ea.row_slot = c->row_slot;
  ea.cos_t = c->cos_t;
  ea.sin_t = c->sin_t;
  ea.max_pos = c->max_pos;
  ea.kv = c->kv;
  ea.x = c->x;
  ea.d = d;
  ea.xn = (bf16*)c->xn;
  ea.ld_xn = xn_ld;
  ea.ss_out = c->ss;
  ea.F = F;
  ea.h = (bf16*)c->xn;
  ea.status = c->d_status;
  ea.lr.row_gate = c->row_gate;

  // DUMP-mode GEMM over X [M, K]: the base segments, then (draft pass) the
  // LoRA A matrices of the same projections as extra output tiles
  auto gemm = [&](const void* X, int ldx, int K, std::initializer_list<std::pair<const void*, int>> w,
                  std::initializer_list<const void*> A, PartView* pv) -> int {
    Gemm g(X, ldx, M, K);
    for (const auto& e : w) g.seg(e.first, e.second);
    const int n_base = g.p.N;
    if (lora)
      for (const void* a : A) g.seg(a, r);
    g.p.lo_off = lo;
    g.p.dep = dep;
    g.p.dep_count = dep ? dep_n + c->dep_extra : dep_n;
    g.p.dep_limit_ns = c->dep_limit_ns;
    g.p.done = next_ctr();
    DumpShape sh;
    {
      Prof prof(c, UNO_K_GEMM, gemm_bytes(g.p, 2) - (double)M * g.p.N * 2, M, g.p.N, K, 0);
      if (!gemm_run_dump(c->genv, g.p, st, &sh))
        return fail(c, UNO_ERR_UNSUPPORTED, "tensor-core GEMM rejected a layer projection");
    }
    *pv = PartView{c->genv.part, sh.NT, sh.units, sh.grid, sh.KBt, sh.m_tiles};
    ea.lr.u_tile0 = n_base / TC_BM;
    dep = g.p.done;
    dep_n = (unsigned)sh.grid;
    return UNO_OK;
  };
  auto set_lora = [&](std::initializer_list<std::pair<const void*, int>> b) {
    ea.lora = lora ? 1 : 0;
    ea.lr.nseg = 0;
    int n0 = 0;
    for (const auto& e : b) {
      ea.lr.Bl[ea.lr.nseg] = (const bf16*)e.first;
      ea.lr.seg_n0[ea.lr.nseg] = n0;
      n0 += e.second;
      ea.lr.nseg++;
    }
  };
  // one epilogue launch: rg rows per CTA (row groups inside the GEMM's
  // m-tiles), `threads` threads
  // `signal`: the next kernel waits on this one's counter
  auto epi = [&](void (*kernel)(const EpiArgs), int tiles, int rg, int threads, bool signal) {
    Prof prof(c, UNO_K_OTHER, 0.0);
    const int groups = ea.pv.m_tiles * epi_groups_per_tile(ea.pv.NT, M, rg);
    ea.dep = dep;
    ea.dep_count = dep ? dep_n + c->dep_extra : 0u;
    ea.dep_limit_ns = c->dep_limit_ns;
    ea.done = signal ? next_ctr() : nullptr;
    dep = ea.done;
    dep_n = (unsigned)(tiles * groups);
    klaunch(pdl, st, dim3(tiles, groups), dim3(threads), 0, kernel, ea);
  };

  {
    static bool co_qkv[ATTR_DEVS] = {}, co_resid[ATTR_DEVS] = {}, co_swiglu[ATTR_DEVS] = {};
    carveout_once(epi_qkv_kernel, co_qkv);
    carveout_once(epi_resid_kernel, co_resid);
    carveout_once(epi_swiglu_kernel, co_swiglu);
  }
  // layer-0 input: g * x and the sums of squares of the embedding rows
  ea.prep = 1;
  ea.lora = 0;
  ea.pv = PartView{nullptr, M, 0, 1, 1, 1};
  ea.g_next = (const bf16*)c->attn_norm[0];
  epi(epi_resid_kernel, d / TC_BM, GeoResid::RG, RESID_THREADS, true);
  ea.prep = 0;

  for (int l = 0; l < s.n_layers; ++l) {
    ea.layer = l;
    int rc = gemm(c->xn, xn_ld, d,
                  {{c->w[UNO_PROJ_Q][l], H * hd}, {c->w[UNO_PROJ_K][l], Hkv * hd},
                   {c->w[UNO_PROJ_V][l], Hkv * hd}},
                  {c->lA[UNO_PROJ_Q][l], c->lA[UNO_PROJ_K][l], c->lA[UNO_PROJ_V][l]}, &ea.pv);
    if (rc) return rc;
    set_lora({{c->lB[UNO_PROJ_Q][l], H * hd}, {c->lB[UNO_PROJ_K][l], Hkv * hd},
              {c->lB[UNO_PROJ_V][l], Hkv * hd}});
    ea.ss = c->ss;
    epi(epi_qkv_kernel, qkv_n / TC_BM, GeoQkv::RG, GeoQkv::THREADS, true);

    // the o GEMM waits for the attention merge with the grid wait (its CTAs
    // start only as the attention CTAs leave the SMs; measured, a counter
    // poll completed later); while the attention streams K/V, its idle lanes
    // pull the first half of W_o into L2 (measured per step at 5120: all of
    // it 8.47 ms, half 8.39, a quarter 8.40, none 8.42: more prefetch traffic
    // slows the epilogue and attention beside it more than it saves)
    AttnSync as;
    as.dep = dep;
    as.dep_n = dep_n;
    as.done = next_ctr();
    rc = launch_attn<bf16>(c, l, n_req, rows_per_req, kind != PASS_PREFILL, attn_lo,
                           c->w[UNO_PROJ_O][l], (size_t)d * hhd, as);
    if (rc) return rc;
    dep = nullptr;

    rc = gemm(c->attn, hhd, hhd, {{c->w[UNO_PROJ_O][l], d}}, {c->lA[UNO_PROJ_O][l]}, &ea.pv);
    if (rc) return rc;
    set_lora({{c->lB[UNO_PROJ_O][l], d}});
    ea.ss = nullptr;
    ea.g_next = (const bf16*)c->ffn_norm[l];
    epi(epi_resid_kernel, d / TC_BM, GeoResid::RG, RESID_THREADS, true);

    rc = gemm(c->xn, xn_ld, d, {{c->w[UNO_PROJ_GATE][l], F}, {c->w[UNO_PROJ_UP][l], F}},
              {c->lA[UNO_PROJ_GATE][l], c->lA[UNO_PROJ_UP][l]}, &ea.pv);
    if (rc) return rc;
    set_lora({{c->lB[UNO_PROJ_GATE][l], F}, {c->lB[UNO_PROJ_UP][l], F}});
    ea.ss = c->ss;
    epi(epi_swiglu_kernel, F / TC_BM, GeoResid::RG, RESID_THREADS, true);

    rc = gemm(c->xn, F, F, {{c->w[UNO_PROJ_DOWN][l], d}}, {c->lA[UNO_PROJ_DOWN][l]}, &ea.pv);
    if (rc) return rc;
    set_lora({{c->lB[UNO_PROJ_DOWN][l], d}});
    ea.ss = nullptr;
    ea.g_next = l + 1 < s.n_layers ? (const bf16*)c->attn_norm[l + 1] : nullptr;
    epi(epi_resid_kernel, d / TC_BM, GeoResid::RG, RESID_THREADS, l + 1 < s.n_layers);
  }
  if (logits) {
    bf16* xn_lo = split ? (bf16*)c->xn + (size_t)lo * xn_ld : nullptr;
    {
      Prof prof(c, UNO_K_OTHER, 0.0);
      klaunch(pdl, st, dim3(M), dim3(256), 0, rmsnorm_kernel<bf16, 256>, (const float*)c->x,
              (const bf16*)c->final_norm, (bf16*)c->xn, xn_lo, d, xn_ld, s.rms_eps);
    }
    Gemm g(c->xn, xn_ld, M, d);
    g.seg(c->lm_head, s.vocab).epi(EPI_STORE_F32, logits, s.vocab, 1.0f / s.temperature);
    g.p.lo_off = lo;
    g.p.out_row = kind == PASS_COHORT ? c->coh_rowoff : nullptr;
    launch_gemm<bf16>(c, g, st);
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

int forward_any(uno_ctx* c, int kind, int n_req, int rows_per_req, const int32_t* req_ids,
                const int32_t* prompt, int prefill_slot, int prefill_pos0, float* logits) {
  // The fused pipeline is built for memory-bound passes (its epilogues are
  // sized for a few dozen rows, one 16-row MMA tile of LoRA-B per CTA); a
  // pass larger than one GEMM token tile runs the unfused kernels, where
  // LoRA-B is a K extension of the tensor-core GEMM and the row kernels are
  // bandwidth-bound.
  if (c->fused && c->fused_enabled && n_req * rows_per_req <= FUSED_MAX_ROWS)
    return forward_fused(c, kind, n_req, rows_per_req, req_ids, prompt, prefill_slot, prefill_pos0,
                         logits);
  if (c->s.dtype == UNO_BF16)
    return forward<bf16>(c, kind, n_req, rows_per_req, req_ids, prompt, prefill_slot, prefill_pos0,
                         logits);
  return forward<float>(c, kind, n_req, rows_per_req, req_ids, prompt, prefill_slot, prefill_pos0,
                        logits);
}

void chunking(int V, int* ch, int* nch) {
  int c = V < 8192 ? ((V + 3) / 4) * 4 : 8192;
  *ch = c;
  *nch = (V + c - 1) / c;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* uno_last_error(const uno_ctx* ctx) { return ctx ? ctx->err.c_str() : "null context"; }

int uno_init(const uno_shape* shape, const uno_weights* wts, int lora_rank, float lora_alpha,
             int block_B, int max_batch, int max_ctx, uint64_t seed, uno_stream_t stream,
             uno_ctx** out) {
  if (!shape || !wts || !out) return UNO_ERR_ARG;
  *out = nullptr;
  const uno_shape& s = *shape;
  if (s.n_layers < 1 || s.d_model < 1 || s.n_heads < 1 || s.n_kv_heads < 1 ||
      s.n_heads % s.n_kv_heads || s.head_dim < 2 || s.ffn_dim < 1 || s.vocab < 2 ||
      s.mask_id < 0 || s.mask_id >= s.vocab || lora_rank < 1 || block_B < 2 || block_B > 64 ||
      max_batch < 1 || max_ctx < 2 || !(s.temperature > 0.f) ||
      (s.dtype != UNO_F32 && s.dtype != UNO_BF16))
    return UNO_ERR_ARG;
  const int G = s.n_heads / s.n_kv_heads;
  const int vec = s.dtype == UNO_BF16 ? 8 : 4;
  if (G > ATT_MAXQ || s.vocab % 4 || s.vocab > MAX_VOCAB || s.d_model % vec || s.ffn_dim % vec ||
      s.d_model > 4 * 256 * RMS_V ||
      lora_rank % vec ||
      (s.n_heads * s.head_dim) % vec ||
      (s.head_dim != 16 && s.head_dim != 32 && s.head_dim != 64 && s.head_dim != 128))
    return UNO_ERR_UNSUPPORTED;
  if (!wts->embed || !wts->lm_head || !wts->final_norm || !wts->attn_norm || !wts->ffn_norm)
    return UNO_ERR_ARG;
  for (int p = 0; p < UNO_N_PROJ; ++p)
    if (!wts->w[p] || !wts->lora_A[p] || !wts->lora_B[p]) return UNO_ERR_ARG;

  uno_ctx* c = new uno_ctx();
  c->s = s;
  c->r = lora_rank;
  c->alpha = lora_alpha;
  c->lscale = lora_alpha / (float)lora_rank;
  c->B = block_B;
  c->max_batch = max_batch;
  c->max_ctx = max_ctx;
  c->seed = seed;
  c->stream = (cudaStream_t)stream;
  c->esz = s.dtype == UNO_BF16 ? 2 : 4;
  c->embed = wts->embed;
  c->lm_head = wts->lm_head;
  c->final_norm = wts->final_norm;
  const int L = s.n_layers;
  c->attn_norm.assign(wts->attn_norm, wts->attn_norm + L);
  c->ffn_norm.assign(wts->ffn_norm, wts->ffn_norm + L);
  for (int p = 0; p < UNO_N_PROJ; ++p) {
    c->w[p].assign(wts->w[p], wts->w[p] + L);
    c->lA[p].assign(wts->lora_A[p], wts->lora_A[p] + L);
    c->lB[p].assign(wts->lora_B[p], wts->lora_B[p] + L);
    for (int l = 0; l < L; ++l)
      if (!c->w[p][l] || !c->lA[p][l] || !c->lB[p][l]) {
        delete c;
        return UNO_ERR_ARG;
      }
  }

  auto oom = [&](const char* what) {
    std::string m = std::string("allocation failed: ") + what;
    uno_destroy(c);
    (void)m;
    return UNO_ERR_OOM;
  };
  const int H = s.n_heads, Hkv = s.n_kv_heads, hd = s.head_dim, d = s.d_model, F = s.ffn_dim;
  const int V = s.vocab, B = block_B;

  // KV pool
  const int ppr = ceil_div(max_ctx + B + 2, KV_PAGE);
  const int n_pages = max_batch * ppr;
  // planes per page: K, V (fp32 models) or K hi, K lo, V in fp16 (bf16 models)
  const int planes = s.dtype == UNO_BF16 ? 3 : 2;
  const size_t kv_bytes = (size_t)L * n_pages * planes * Hkv * KV_PAGE * hd * c->esz;
  if (dalloc(&c->kv_pool, kv_bytes) != cudaSuccess) return oom("kv pool");
  // zeroed: keys past a request's length are masked out of the scores, and
  // the values there must be finite so that P V (with P = 0) stays finite
  cudaMemset(c->kv_pool, 0, kv_bytes);
  // page-table rows: the request slots, then the tree sampler's chain slots
  const size_t pt_rows = (size_t)max_batch * (1 + TREE_MAX_K);
  if (dalloc(&c->d_page_table, pt_rows * ppr * 4) != cudaSuccess) return oom("pages");
  if (dalloc(&c->d_cached, (size_t)max_batch * 4) != cudaSuccess) return oom("state");
  if (dalloc(&c->d_pending, (size_t)max_batch * 4) != cudaSuccess) return oom("state");
  if (dalloc(&c->d_stream, (size_t)max_batch * 4) != cudaSuccess) return oom("state");
  c->kv = KvLayout{c->kv_pool, n_pages, Hkv, hd, ppr, c->d_page_table, planes};
  c->free_pages.resize(n_pages);
  for (int i = 0; i < n_pages; ++i) c->free_pages[i] = n_pages - 1 - i;
  c->slot_used.assign(max_batch, 0);
  c->h_page_table.assign((size_t)max_batch * ppr, 0);
  cudaMemset(c->d_page_table, 0, pt_rows * ppr * 4);
  cudaMemset(c->d_cached, 0, (size_t)max_batch * 4);
  cudaMemset(c->d_pending, 0, (size_t)max_batch * 4);
  cudaMemset(c->d_stream, 0, (size_t)max_batch * 4);

  // activations
  const int M = std::max(max_batch * (B + 1), PREFILL_CHUNK);
  c->M_max = M;
  const size_t e = c->esz;
  if (dalloc(&c->x, (size_t)M * d * 4) != cudaSuccess) return oom("x");
  if (dalloc(&c->xn, (size_t)2 * M * std::max(d, F) * e) != cudaSuccess) return oom("xn");
  if (dalloc(&c->qkv, (size_t)M * (H + 2 * Hkv) * hd * 4) != cudaSuccess) return oom("qkv");
  // q rows: hi rows [0, M), lo rows (bf16 models) from M_max on
  if (dalloc(&c->qbuf, (size_t)2 * M * H * hd * e) != cudaSuccess) return oom("q");
  cudaMemset(c->qbuf, 0, (size_t)2 * M * H * hd * e);
  if (dalloc(&c->attn, (size_t)2 * M * H * hd * e) != cudaSuccess) return oom("attn");
  if (dalloc(&c->gu, (size_t)M * 2 * F * 4) != cudaSuccess) return oom("gu");
  if (dalloc(&c->U, (size_t)2 * M * 3 * lora_rank * e) != cudaSuccess) return oom("U");
  if (dalloc(&c->row_pos, (size_t)M * 4) != cudaSuccess) return oom("rows");
  if (dalloc(&c->row_slot, (size_t)M * 4) != cudaSuccess) return oom("rows");
  if (dalloc(&c->row_gate, (size_t)M * 4) != cudaSuccess) return oom("rows");
  if (dalloc(&c->row_cslot, (size_t)M * 4) != cudaSuccess) return oom("rows");
  if (dalloc(&c->row_blk, (size_t)M * 4) != cudaSuccess) return oom("rows");
  if (dalloc(&c->train_slots, (size_t)2 * max_batch * 4) != cudaSuccess) return oom("rows");
  c->n_dep_ctr = 10 * s.n_layers + 8;
  if (dalloc(&c->dep_ctr, (size_t)c->n_dep_ctr * 4) != cudaSuccess) return oom("counters");
  cudaMemset(c->dep_ctr, 0, (size_t)c->n_dep_ctr * 4);

  // RoPE table, double precision on the host
  c->max_pos = ppr * KV_PAGE;
  {
    const int half = hd / 2;
    std::vector<float> ct((size_t)c->max_pos * half), stb((size_t)c->max_pos * half);
    for (int pos = 0; pos < c->max_pos; ++pos)
      for (int i = 0; i < half; ++i) {
        const double inv = std::pow((double)s.rope_theta, -2.0 * i / hd);
        const double a = (double)pos * inv;
        ct[(size_t)pos * half + i] = (float)std::cos(a);
        stb[(size_t)pos * half + i] = (float)std::sin(a);
      }
    if (dalloc(&c->cos_t, ct.size() * 4) != cudaSuccess) return oom("rope");
    if (dalloc(&c->sin_t, ct.size() * 4) != cudaSuccess) return oom("rope");
    cudaMemcpy(c->cos_t, ct.data(), ct.size() * 4, cudaMemcpyHostToDevice);
    cudaMemcpy(c->sin_t, stb.data(), stb.size() * 4, cudaMemcpyHostToDevice);
  }

  // logits and sampler workspaces
  chunking(V, &c->ch, &c->nch);
  if (dalloc(&c->logits_d, (size_t)max_batch * (B + 1) * V * 4) != cudaSuccess) return oom("logits");
  if (dalloc(&c->logits_v, (size_t)max_batch * B * V * 4) != cudaSuccess) return oom("logits");
  if (dalloc(&c->drafts, (size_t)max_batch * B * 4) != cudaSuccess) return oom("drafts");
  if (dalloc(&c->lse_q, (size_t)max_batch * B * 4) != cudaSuccess) return oom("lse");
  // sampled / reduced rows per request: 2B (verify), 1 + k (B - 1) (tree drafts)
  const size_t rows_ws = (size_t)max_batch * std::max(2 * B, 1 + TREE_MAX_K * (B - 1));
  if (dalloc(&c->partial, rows_ws * c->nch * sizeof(float2)) != cudaSuccess) return oom("partial");
  if (dalloc(&c->lse_ws, rows_ws * 4) != cudaSuccess) return oom("lse");
  if (dalloc(&c->row_counter, rows_ws * 4) != cudaSuccess) return oom("counters");
  if (dalloc(&c->req_counter, (size_t)max_batch * 4) != cudaSuccess) return oom("counters");
  if (dalloc(&c->at_ws, (size_t)max_batch * 4) != cudaSuccess) return oom("verify ws");
  if (dalloc(&c->filt_d, (size_t)max_batch * (B + 1) * sizeof(RowFilter)) != cudaSuccess) return oom("filters");
  if (dalloc(&c->filt_v, (size_t)max_batch * B * sizeof(RowFilter)) != cudaSuccess) return oom("filters");
  cudaMemset(c->filt_d, 0, (size_t)max_batch * (B + 1) * sizeof(RowFilter));
  cudaMemset(c->filt_v, 0, (size_t)max_batch * B * sizeof(RowFilter));
  if (dalloc(&c->resid_part, (size_t)max_batch * c->nch * 4) != cudaSuccess) return oom("verify ws");
  if (dalloc(&c->resid_counter, (size_t)max_batch * 4) != cudaSuccess) return oom("counters");
  cudaMemset(c->row_counter, 0, rows_ws * 4);
  cudaMemset(c->req_counter, 0, (size_t)max_batch * 4);
  cudaMemset(c->resid_counter, 0, (size_t)max_batch * 4);
  cudaMemset(c->drafts, 0, (size_t)max_batch * B * 4);

  // attention split workspace: groups x splits <= about two waves of CTAs
  c->att_groups_max = max_batch * Hkv * ceil_div(B + 1, ATT_MAXQ / (H / Hkv));
  c->att_ws_floats = (size_t)(2 * 148 + c->att_groups_max) * ATC_QROWS * atc_ws_row(hd);
  if (dalloc(&c->att_ws, c->att_ws_floats * 4) != cudaSuccess) return oom("attention ws");
  if (dalloc(&c->att_counters, (size_t)c->att_groups_max * 4) != cudaSuccess) return oom("attention ws");
  cudaMemset(c->att_counters, 0, (size_t)c->att_groups_max * 4);
  if (dalloc(&c->d_status, 4) != cudaSuccess) return oom("status");
  cudaMemset(c->d_status, 0, 4);

  // tensor-core GEMM: one persistent CTA per SM, partial tiles, counters
  {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    c->genv.sm_count = sms;
    c->genv.pdl = true;
    c->genv.x_rows_alloc = 2 * M;   // activation buffers: hi rows then lo rows
    if (dalloc(&c->genv.ws, GemmEnv::ws_bytes(sms)) != cudaSuccess) return oom("gemm ws");
    if (dalloc(&c->genv.counters, (size_t)TC_COUNTERS * 4) != cudaSuccess) return oom("gemm ws");
    cudaMemset(c->genv.counters, 0, (size_t)TC_COUNTERS * 4);
    c->genv.status = c->d_status;
  }
  // fused bf16 layer pipeline: 128-column tiles must not straddle q/k/v or
  // heads, the adapter rank must fill whole tiles, weights 16-byte aligned
  {
    bool ok = s.dtype == UNO_BF16 && (hd == 64 || hd == 128) && d % TC_BM == 0 &&
              F % TC_BM == 0 && (H * hd) % TC_BM == 0 && (Hkv * hd) % TC_BM == 0 &&
              (lora_rank == 0 || lora_rank == EPI_R) && d <= EPI_MAX_SS * TC_BM;
    for (int pj = 0; pj < UNO_N_PROJ && ok; ++pj)
      for (int l = 0; l < L && ok; ++l) {
        ok = ((uintptr_t)c->w[pj][l] & 15) == 0;
        if (lora_rank) ok = ok && ((uintptr_t)c->lA[pj][l] & 15) == 0 && ((uintptr_t)c->lB[pj][l] & 15) == 0;
      }
    if (ok) {
      size_t part = 0;
      const int rr = lora_rank;
      for (int m = 1; m <= M; ++m) {
        const int ns[4] = {(H + 2 * Hkv) * hd + 3 * rr, d + rr, 2 * F + 2 * rr, d + rr};
        for (int k = 0; k < 4; ++k)
          part = std::max(part, dump_bytes(m, ns[k], c->genv.sm_count, /*split=*/true));
      }
      if (dalloc(&c->genv.part, part) != cudaSuccess) return oom("gemm parts");
      c->genv.part_bytes = part;
      if (dalloc(&c->ss, (size_t)M * (d / TC_BM) * 4) != cudaSuccess) return oom("norm sums");
      c->fused = true;
    }
  }
  // tensor-core attention: the pool (fp16 for bf16 models) as a [rows, head_dim]
  // tensor, 64x64 boxes.  Its kernel forms pool rows and TMA coordinates as
  // 32-bit ints: a pool of 2^31 rows or more (about 270 requests of 9232
  // tokens on the Qwen3-8B shape) takes the SIMT attention instead.
  const uint64_t kv_rows = (uint64_t)L * n_pages * planes * Hkv * KV_PAGE;
  if (s.dtype == UNO_BF16 && (hd == 64 || hd == 128) && ATC_QROWS % G == 0 &&
      kv_rows < ((uint64_t)1 << 31)) {
    const uint64_t rows = kv_rows;
    const CUtensorMap* m = c->genv.map(c->kv_pool, rows, hd, hd, KV_PAGE, /*fp16=*/true);
    // q: box (64 of head_dim, the G heads of a kv head, the query tile's tokens)
    EncodeTiledFn f = encode_fn();
    const cuuint64_t qdims[3] = {(cuuint64_t)hd, (cuuint64_t)H, (cuuint64_t)2 * M};
    const cuuint64_t qstrides[2] = {(cuuint64_t)hd * 2, (cuuint64_t)H * hd * 2};
    const cuuint32_t qbox[3] = {64, (cuuint32_t)G, (cuuint32_t)(ATC_QROWS / G)};
    const cuuint32_t qes[3] = {1, 1, 1};
    const bool qok = f && f(&c->q_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, c->qbuf, qdims, qstrides,
                            qbox, qes, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    if (m && qok) {
      c->kv_map = *m;
      c->kv_map_ok = true;
    }
  }
  if (cudaDeviceSynchronize() != cudaSuccess) {
    uno_destroy(c);
    return UNO_ERR_CUDA;
  }
  *out = c;
  return UNO_OK;
}

int uno_destroy(uno_ctx* c) {
  if (!c) return UNO_ERR_ARG;
  if (c->stream) cudaStreamSynchronize(c->stream);
  cudaDeviceSynchronize();
  void* bufs[] = {c->kv_pool, c->d_page_table, c->d_cached, c->d_pending, c->d_stream, c->x,
                  c->xn, c->qkv, c->qbuf, c->attn, c->gu, c->U, c->row_pos, c->row_slot, c->row_gate,
                  c->row_cslot, c->row_blk, c->train_slots, c->coh_logits, c->coh_drafts,
                  c->coh_lse_q, c->coh_phase, c->coh_rows, c->coh_rowoff, c->logits_t,
                  c->lse_t, c->tree_chains, c->tree_resid, c->tree_walk, c->tree_pages,
                  c->dep_ctr, c->cos_t, c->sin_t, c->logits_d, c->logits_v, c->drafts, c->lse_q, c->partial,
                  c->lse_ws, c->row_counter, c->req_counter, c->at_ws, c->resid_part,
                  c->resid_counter, c->att_ws, c->att_counters, c->filt_d, c->filt_v,
                  c->d_status, c->genv.ws, c->genv.counters, c->genv.part, c->ss};
  for (void* b : bufs)
    if (b) cudaFree(b);
  for (cudaEvent_t e : c->ev_pool) cudaEventDestroy(e);
  for (auto& g : c->graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (c->cap_stream) cudaStreamDestroy(c->cap_stream);
  delete c;
  return UNO_OK;
}

int uno_prefill(uno_ctx* c, int n_req, const int32_t* prompts_dev, int prompt_stride,
                const int32_t* prompt_lens_host, const uint32_t* streams_host,
                int32_t* req_ids_host_out) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_req < 1 || !prompts_dev || !prompt_lens_host || !req_ids_host_out || prompt_stride < 1)
    return fail(c, UNO_ERR_ARG, "bad prefill arguments");
  int free_slots = 0;
  for (int u : c->slot_used) free_slots += !u;
  const int ppr = c->kv.pages_per_req;
  if (free_slots < n_req || (int)c->free_pages.size() < n_req * ppr)
    return fail(c, UNO_ERR_CAPACITY, "no free request slot or KV pages");
  for (int i = 0; i < n_req; ++i)
    if (prompt_lens_host[i] < 1 || prompt_lens_host[i] > c->max_ctx || prompt_lens_host[i] > prompt_stride)
      return fail(c, UNO_ERR_ARG, "prompt length out of range");
  for (int i = 0; i < n_req; ++i) {
    int slot = 0;
    while (c->slot_used[slot]) ++slot;
    c->slot_used[slot] = 1;
    for (int pi = 0; pi < ppr; ++pi) {
      c->h_page_table[(size_t)slot * ppr + pi] = c->free_pages.back();
      c->free_pages.pop_back();
    }
    CK(cudaMemcpyAsync(c->d_page_table + (size_t)slot * ppr, c->h_page_table.data() + (size_t)slot * ppr,
                       ppr * 4, cudaMemcpyHostToDevice, c->stream));
    const uint32_t sid = streams_host ? streams_host[i] : (uint32_t)slot;
    CK(cudaMemcpyAsync(c->d_stream + slot, &sid, 4, cudaMemcpyHostToDevice, c->stream));
    CK(cudaStreamSynchronize(c->stream));  // host staging values above are locals
    req_ids_host_out[i] = slot;
    const int P = prompt_lens_host[i];
    const int32_t* prompt = prompts_dev + (size_t)i * prompt_stride;
    for (int p0 = 0; p0 < P - 1; p0 += PREFILL_CHUNK) {
      const int n = std::min(PREFILL_CHUNK, P - 1 - p0);
      const int rc = forward_any(c, PASS_PREFILL, 1, n, nullptr, prompt + p0, slot, p0, nullptr);
      if (rc) return rc;
    }
    init_slot_kernel<<<1, 1, 0, c->stream>>>(prompt, P, slot, c->d_cached, c->d_pending);
    CK(cudaGetLastError());
    // a new request starts undrafted for the cohort step
    if (c->coh_phase) CK(cudaMemsetAsync(c->coh_phase + slot, 0, 4, c->stream));
  }
  return UNO_OK;
}

int uno_train_forward(uno_ctx* c, int n_seq, const int32_t* tokens_dev, int L, float* logits_dev) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_seq < 1 || L < 1 || !tokens_dev || !logits_dev)
    return fail(c, UNO_ERR_ARG, "bad train_forward arguments");
  if ((long long)n_seq * 2 * L > c->M_max)
    return fail(c, UNO_ERR_CAPACITY, "n_seq * 2L rows exceed the pass capacity");
  if (L > c->max_ctx) return fail(c, UNO_ERR_ARG, "L exceeds max_ctx");
  int free_slots = 0;
  for (int u : c->slot_used) free_slots += !u;
  const int ppr = c->kv.pages_per_req;
  if (free_slots < 2 * n_seq || (int)c->free_pages.size() < 2 * n_seq * ppr)
    return fail(c, UNO_ERR_CAPACITY, "no free request slots or KV pages for the training form");
  // two slots per sequence: clean keys, noised keys (positions 0 .. L-1 each)
  std::vector<int32_t> slots;
  for (int i = 0; i < 2 * n_seq; ++i) {
    int slot = 0;
    while (c->slot_used[slot]) ++slot;
    c->slot_used[slot] = 1;
    for (int pi = 0; pi < ppr; ++pi) {
      c->h_page_table[(size_t)slot * ppr + pi] = c->free_pages.back();
      c->free_pages.pop_back();
    }
    slots.push_back(slot);
  }
  auto release = [&]() {
    for (int slot : slots) {
      for (int pi = 0; pi < ppr; ++pi) c->free_pages.push_back(c->h_page_table[(size_t)slot * ppr + pi]);
      c->slot_used[slot] = 0;
    }
  };
  for (int slot : slots) {
    const cudaError_t e = cudaMemcpyAsync(c->d_page_table + (size_t)slot * ppr,
                                          c->h_page_table.data() + (size_t)slot * ppr, ppr * 4,
                                          cudaMemcpyHostToDevice, c->stream);
    if (e != cudaSuccess) { release(); return fail(c, UNO_ERR_CUDA, cudaGetErrorString(e)); }
  }
  cudaError_t e = cudaMemcpyAsync(c->train_slots, slots.data(), slots.size() * 4,
                                  cudaMemcpyHostToDevice, c->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->stream);   // host staging above is local
  if (e != cudaSuccess) { release(); return fail(c, UNO_ERR_CUDA, cudaGetErrorString(e)); }
  const int rc = forward_any(c, PASS_TRAIN, n_seq, 2 * L, c->train_slots, tokens_dev, 0, 0, logits_dev);
  // later work on the stream runs after this pass, so the slots can be reused
  release();
  return rc;
}

}  // extern "C"

namespace {

// Runs body() eagerly on the first call with a given argument set (which
// also creates descriptors and kernel attributes), captures it into a CUDA
// graph on the second call and replays the graph from then on.  Profiling
// runs eagerly (its event pairs are host-side bookkeeping).
template <typename F>
int run_graphed(uno_ctx* c, int kind, int n_req, const void* a, const void* b, const void* d,
                F&& body, const void* d2 = nullptr) {
  if (!c->graphs_enabled || c->prof_mask) return body();
  uno_ctx::GraphEntry* e = nullptr;
  for (auto& g : c->graphs)
    if (g.kind == kind && g.n_req == n_req && g.a == a && g.b == b && g.c == d && g.d == d2) e = &g;
  if (!e) {
    c->graphs.emplace_back();
    e = &c->graphs.back();
    e->kind = kind; e->n_req = n_req; e->a = a; e->b = b; e->c = d; e->d = d2;
  }
  if (e->exec) {
    CK(cudaGraphLaunch(e->exec, c->stream));
    for (int k = 0; k < UNO_K_N; ++k) {
      c->prof_launches[k] += e->launches[k];
      c->prof_bytes[k] += e->bytes[k];
    }
    for (int i = 0; i < 4; ++i) g_launches[i] += e->glaunch[i];
    return UNO_OK;
  }
  if (e->seen++ == 0) return body();
  if (!c->cap_stream) CK(cudaStreamCreateWithFlags(&c->cap_stream, cudaStreamNonBlocking));
  int64_t l0[UNO_K_N], g0[4];
  double b0[UNO_K_N];
  for (int k = 0; k < UNO_K_N; ++k) { l0[k] = c->prof_launches[k]; b0[k] = c->prof_bytes[k]; }
  for (int i = 0; i < 4; ++i) g0[i] = g_launches[i];
  cudaStream_t user = c->stream;
  c->stream = c->cap_stream;
  cudaError_t ce = cudaStreamBeginCapture(c->cap_stream, cudaStreamCaptureModeThreadLocal);
  if (ce != cudaSuccess) {
    c->stream = user;
    return fail(c, UNO_ERR_CUDA, std::string("begin capture: ") + cudaGetErrorString(ce));
  }
  const int rc = body();
  cudaGraph_t graph = nullptr;
  ce = cudaStreamEndCapture(c->cap_stream, &graph);
  c->stream = user;
  if (rc != UNO_OK || ce != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return rc != UNO_OK ? rc : fail(c, UNO_ERR_CUDA, std::string("end capture: ") + cudaGetErrorString(ce));
  }
  ce = cudaGraphInstantiate(&e->exec, graph, 0);
  cudaGraphDestroy(graph);
  if (ce != cudaSuccess) {
    e->exec = nullptr;
    return fail(c, UNO_ERR_CUDA, std::string("instantiate: ") + cudaGetErrorString(ce));
  }
  for (int k = 0; k < UNO_K_N; ++k) {
    e->launches[k] = c->prof_launches[k] - l0[k];
    e->bytes[k] = c->prof_bytes[k] - b0[k];
  }
  for (int i = 0; i < 4; ++i) e->glaunch[i] = g_launches[i] - g0[i];
  CK(cudaGraphLaunch(e->exec, c->stream));   // counted once, by the capture above
  return UNO_OK;
}

// The tree sampler's iteration (tree_k >= 2): the draft pass, k drafted
// chains, one verify pass over every chain, the walk and the commit.
int tree_step_body(uno_ctx* c, int n_req, const int32_t* req_ids_dev, int32_t* out_tokens_dev,
                   int32_t* n_new_dev) {
  const int B = c->B, V = c->s.vocab, k = c->tree_k;
  int rc = forward_any(c, PASS_DRAFT, n_req, B + 1, req_ids_dev, nullptr, 0, 0, c->logits_d);
  if (rc) return rc;
  const int rows = 1 + k * (B - 1);
  {
    SampleArgs a{};
    a.logits = c->logits_d;
    a.V = V; a.nch = c->nch; a.ch = c->ch;
    a.rows_per_req = rows;
    a.logit_rows_per_req = B + 1;
    a.ar_mode = 0;
    a.req_slot = req_ids_dev;
    a.cached = c->d_cached;
    a.pending = c->d_pending;
    a.slot_stream = c->d_stream;
    a.seed = c->seed;
    a.out_tok = c->tree_chains;
    a.out_stride = B;
    a.lse_out = c->lse_q;
    a.partial = c->partial;
    a.row_counter = c->row_counter;
    a.status = c->d_status;
    a.tree_k = k;
    a.tree_B = B;
    Prof prof(c, UNO_K_SAMPLE, (double)n_req * rows * V * 4);
    launch_sample(c->genv.pdl, c->stream, dim3(c->nch, n_req * rows), a);
  }
  rc = forward_any(c, PASS_TREE, n_req * k, B, req_ids_dev, nullptr, 0, 0, c->logits_t);
  if (rc) return rc;
  {
    Prof prof(c, UNO_K_VERIFY, (double)n_req * k * B * V * 4);
    klaunch(c->genv.pdl, c->stream, dim3(n_req * k * B), dim3(TREE_THREADS), 0, row_lse_kernel,
            (const float*)c->logits_t, V, c->lse_t);
  }
  {
    TreeArgs a{};
    a.q = c->logits_d; a.lse_q = c->lse_q;
    a.p = c->logits_t; a.lse_p = c->lse_t;
    a.chains = c->tree_chains;
    a.V = V; a.B = B; a.k = k;
    a.seed = c->seed;
    a.req_slot = req_ids_dev;
    a.cached = c->d_cached; a.pending = c->d_pending; a.slot_stream = c->d_stream;
    a.resid = c->tree_resid;
    a.out_tok = out_tokens_dev; a.out_stride = B + 1; a.n_out = n_new_dev;
    a.walk = c->tree_walk;
    a.status = c->d_status;
    Prof prof(c, UNO_K_VERIFY, (double)n_req * 4 * V * 4);
    klaunch(c->genv.pdl, c->stream, dim3(n_req), dim3(TREE_THREADS), 0, tree_walk_kernel, a);
  }
  {
    TreeCommitArgs a{};
    a.kv = c->kv;
    a.max_batch = c->max_batch;
    a.esz = c->s.dtype == UNO_BF16 ? 2 : 4;
    a.req_slot = req_ids_dev;
    a.walk = c->tree_walk;
    a.status = c->d_status;
    Prof prof(c, UNO_K_OTHER, 0.0);
    klaunch(c->genv.pdl, c->stream, dim3(B, c->s.n_layers, n_req), dim3(256), 0, tree_commit_kernel, a);
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

int spec_step_body(uno_ctx* c, int n_req, const int32_t* req_ids_dev, int32_t* out_tokens_dev,
                   int32_t* n_new_dev) {
  if (c->tree_k >= 2) return tree_step_body(c, n_req, req_ids_dev, out_tokens_dev, n_new_dev);
  const int B = c->B, V = c->s.vocab;
  int rc = forward_any(c, PASS_DRAFT, n_req, B + 1, req_ids_dev, nullptr, 0, 0, c->logits_d);
  if (rc) return rc;
  const bool filt = c->top_p < 1.f;
  auto nucleus = [&](const float* logits, int64_t logit_rows, int draft_map, RowFilter* out) -> int {
    TopPArgs t{};
    t.logits = logits; t.V = V; t.rows_per_req = B; t.logit_rows_per_req = logit_rows;
    t.draft_map = draft_map; t.top_p = c->top_p; t.out = out;
    Prof prof(c, UNO_K_SAMPLE, (double)n_req * B * V * 4);
    return launch_top_p(c->genv.pdl, c->stream, t, n_req)
               ? UNO_OK : fail(c, UNO_ERR_CUDA, "top-p kernel attributes");
  };
  // draft rows p_1 (row 0) and q_2..q_B (rows 2..B)
  if (filt && (rc = nucleus(c->logits_d, B + 1, 1, c->filt_d))) return rc;
  {
    SampleArgs a{};
    a.filt = filt ? c->filt_d : nullptr;
    a.logits = c->logits_d;
    a.V = V; a.nch = c->nch; a.ch = c->ch;
    a.rows_per_req = B;
    a.logit_rows_per_req = B + 1;
    a.ar_mode = 0;
    a.req_slot = req_ids_dev;
    a.cached = c->d_cached;
    a.pending = c->d_pending;
    a.slot_stream = c->d_stream;
    a.seed = c->seed;
    a.out_tok = c->drafts;
    a.out_stride = B;
    a.lse_out = c->lse_q;
    a.partial = c->partial;
    a.row_counter = c->row_counter;
    a.status = c->d_status;
    Prof prof(c, UNO_K_SAMPLE, (double)n_req * B * V * 4);
    launch_sample(c->genv.pdl, c->stream, dim3(c->nch, n_req * B), a);
  }
  rc = forward_any(c, PASS_VERIFY, n_req, B, req_ids_dev, nullptr, 0, 0, c->logits_v);
  if (rc) return rc;
  // verify rows p_2..p_{B+1}
  if (filt && (rc = nucleus(c->logits_v, B, 0, c->filt_v))) return rc;
  {
    VerifyArgs a{};
    a.filt_p = filt ? c->filt_v : nullptr;
    a.filt_q = filt ? c->filt_d : nullptr;
    a.p = c->logits_v;
    a.q = c->logits_d;
    a.V = V; a.nch = c->nch; a.ch = c->ch;
    a.n_tests = B - 1;
    a.p_req_rows = B;
    a.q_req_rows = B + 1;
    a.p_row0 = 0;
    a.q_row0 = 2;
    a.bonus_row = B - 1;
    a.drafts = c->drafts; a.drafts_stride = B; a.drafts_off = 1;
    a.lse_q_in = c->lse_q; a.lse_q_stride = B; a.lse_q_off = 1;
    a.seed = c->seed;
    a.req_slot = req_ids_dev;
    a.cached = c->d_cached;
    a.pending = c->d_pending;
    a.slot_stream = c->d_stream;
    a.first_tok = c->drafts;
    a.out_tok = out_tokens_dev;
    a.out_stride = B + 1;
    a.n_out = n_new_dev;
    a.partial = c->partial;
    a.lse = c->lse_ws;
    a.row_counter = c->row_counter;
    a.req_counter = c->req_counter;
    a.at_ws = c->at_ws;
    a.resid_part = c->resid_part;
    a.resid_counter = c->resid_counter;
    a.rows_red = B;      // B - 1 test rows + the bonus row; lse of q comes from draft_sample
    a.n_p = B;
    a.status = c->d_status;
    a.fixed_at = c->fixed_accept > 0 ? c->fixed_accept - 1 : -1;
    {
      Prof prof(c, UNO_K_VERIFY, (double)n_req * B * V * 4);
      c->prof_launches[UNO_K_VERIFY] +=
          launch_verify(c->genv.pdl, c->stream, a, n_req, c->verify_split_ctas, filt) - 1;
    }
    {
      Prof prof(c, UNO_K_VERIFY, (double)n_req * 2 * V * 4);
      launch_resid(c->genv.pdl, c->stream, a, n_req, filt);
    }
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

// One forward over the drafting cohort's draft rows and the verifying
// cohort's verify rows, then draft_sample of the first and spec_verify +
// commit of the second (per-slot state in between).
int cohort_step_body(uno_ctx* c, int n_draft, const int32_t* draft_ids, int n_verify,
                     const int32_t* verify_ids, int32_t* out_tokens, int32_t* n_new) {
  const int B = c->B, V = c->s.vocab;
  const int n = n_draft + n_verify;
  if (n_draft)
    CK(cudaMemcpyAsync(c->coh_rows, draft_ids, (size_t)n_draft * 4, cudaMemcpyDeviceToDevice, c->stream));
  if (n_verify)
    CK(cudaMemcpyAsync(c->coh_rows + n_draft, verify_ids, (size_t)n_verify * 4, cudaMemcpyDeviceToDevice,
                       c->stream));
  c->coh_n_draft = n_draft;
  int rc = forward_any(c, PASS_COHORT, n, B + 1, c->coh_rows, nullptr, 0, 0, c->coh_logits);
  if (rc) return rc;
  if (n_draft) {
    SampleArgs a{};
    a.logits = c->coh_logits;
    a.V = V; a.nch = c->nch; a.ch = c->ch;
    a.rows_per_req = B;
    a.logit_rows_per_req = B + 1;
    a.ar_mode = 0;
    a.req_slot = c->coh_rows;
    a.cached = c->d_cached;
    a.pending = c->d_pending;
    a.slot_stream = c->d_stream;
    a.seed = c->seed;
    a.out_tok = c->coh_drafts;
    a.out_stride = B;
    a.lse_out = c->coh_lse_q;
    a.partial = c->partial;
    a.row_counter = c->row_counter;
    a.status = c->d_status;
    a.per_slot = 1;
    a.phase = c->coh_phase;
    Prof prof(c, UNO_K_SAMPLE, (double)n_draft * B * V * 4);
    launch_sample(c->genv.pdl, c->stream, dim3(c->nch, n_draft * B), a);
  }
  if (n_verify) {
    VerifyArgs a{};
    a.p = c->coh_logits + (size_t)c->max_batch * (B + 1) * V;
    a.q = c->coh_logits;
    a.V = V; a.nch = c->nch; a.ch = c->ch;
    a.n_tests = B - 1;
    a.p_req_rows = B + 1;
    a.q_req_rows = B + 1;
    a.p_row0 = 0;
    a.q_row0 = 2;
    a.bonus_row = B - 1;
    a.drafts = c->coh_drafts; a.drafts_stride = B; a.drafts_off = 1;
    a.lse_q_in = c->coh_lse_q; a.lse_q_stride = B; a.lse_q_off = 1;
    a.seed = c->seed;
    a.req_slot = c->coh_rows + n_draft;
    a.cached = c->d_cached;
    a.pending = c->d_pending;
    a.slot_stream = c->d_stream;
    a.first_tok = c->coh_drafts;
    a.out_tok = out_tokens;
    a.out_stride = B + 1;
    a.n_out = n_new;
    a.partial = c->partial;
    a.lse = c->lse_ws;
    a.row_counter = c->row_counter;
    a.req_counter = c->req_counter;
    a.at_ws = c->at_ws;
    a.resid_part = c->resid_part;
    a.resid_counter = c->resid_counter;
    a.rows_red = B;
    a.n_p = B;
    a.status = c->d_status;
    a.fixed_at = c->fixed_accept > 0 ? c->fixed_accept - 1 : -1;
    a.per_slot = 1;
    a.phase = c->coh_phase;
    {
      Prof prof(c, UNO_K_VERIFY, (double)n_verify * B * V * 4);
      c->prof_launches[UNO_K_VERIFY] +=
          launch_verify(c->genv.pdl, c->stream, a, n_verify, c->verify_split_ctas, false) - 1;
    }
    {
      Prof prof(c, UNO_K_VERIFY, (double)n_verify * 2 * V * 4);
      launch_resid(c->genv.pdl, c->stream, a, n_verify, false);
    }
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

int ar_step_body(uno_ctx* c, int n_req, const int32_t* req_ids_dev, int32_t* out_tokens_dev) {
  int rc = forward_any(c, PASS_AR, n_req, 1, req_ids_dev, nullptr, 0, 0, c->logits_d);
  if (rc) return rc;
  const bool filt = c->top_p < 1.f;
  if (filt) {
    TopPArgs t{};
    t.logits = c->logits_d; t.V = c->s.vocab; t.rows_per_req = 1; t.logit_rows_per_req = 1;
    t.draft_map = 0; t.top_p = c->top_p; t.out = c->filt_d;
    Prof prof(c, UNO_K_SAMPLE, (double)n_req * c->s.vocab * 4);
    if (!launch_top_p(c->genv.pdl, c->stream, t, n_req))
      return fail(c, UNO_ERR_CUDA, "top-p kernel attributes");
  }
  SampleArgs a{};
  a.filt = filt ? c->filt_d : nullptr;
  a.logits = c->logits_d;
  a.V = c->s.vocab; a.nch = c->nch; a.ch = c->ch;
  a.rows_per_req = 1;
  a.logit_rows_per_req = 1;
  a.ar_mode = 1;
  a.req_slot = req_ids_dev;
  a.cached = c->d_cached;
  a.pending = c->d_pending;
  a.slot_stream = c->d_stream;
  a.seed = c->seed;
  a.out_tok = out_tokens_dev;
  a.out_stride = 1;
  a.partial = c->partial;
  a.row_counter = c->row_counter;
  a.status = c->d_status;
  {
    Prof prof(c, UNO_K_SAMPLE, (double)n_req * a.V * 4);
    launch_sample(c->genv.pdl, c->stream, dim3(c->nch, n_req), a);
  }
  CK(cudaGetLastError());
  return UNO_OK;
}

}  // namespace

extern "C" {

int uno_spec_step(uno_ctx* c, int n_req, const int32_t* req_ids_dev, int32_t* out_tokens_dev,
                  int32_t* n_new_dev) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_req < 1 || n_req > c->max_batch || !req_ids_dev || !out_tokens_dev || !n_new_dev)
    return fail(c, UNO_ERR_ARG, "bad spec_step arguments");
  if (c->tree_k >= 2 && (long long)n_req * c->tree_k * c->B > c->M_max)
    return fail(c, UNO_ERR_CAPACITY, "tree verify rows exceed the pass capacity");
  if (c->tree_k >= 2 && c->top_p < 1.f)
    return fail(c, UNO_ERR_UNSUPPORTED, "the tree sampler samples without top-p");
  c->last_n_req = n_req;
  return run_graphed(c, 0, n_req, req_ids_dev, out_tokens_dev, n_new_dev, [&] {
    return spec_step_body(c, n_req, req_ids_dev, out_tokens_dev, n_new_dev);
  });
}

int uno_spec_step_cohorts(uno_ctx* c, int n_draft, const int32_t* draft_ids_dev, int n_verify,
                          const int32_t* verify_ids_dev, int32_t* out_tokens_dev, int32_t* n_new_dev) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_draft < 0 || n_verify < 0 || n_draft + n_verify < 1 || n_draft + n_verify > c->max_batch ||
      (n_draft && !draft_ids_dev) || (n_verify && (!verify_ids_dev || !out_tokens_dev || !n_new_dev)))
    return fail(c, UNO_ERR_ARG, "bad cohort step arguments");
  if (c->top_p < 1.f) return fail(c, UNO_ERR_UNSUPPORTED, "the cohort step samples without top-p");
  if (!c->coh_logits) {
    // first call: the per-slot buffers (one-time allocation)
    const size_t B = c->B, V = c->s.vocab, mb = c->max_batch;
    if (dalloc(&c->coh_logits, 2 * mb * (B + 1) * V * 4) != cudaSuccess ||
        dalloc(&c->coh_drafts, mb * B * 4) != cudaSuccess || dalloc(&c->coh_lse_q, mb * B * 4) != cudaSuccess ||
        dalloc(&c->coh_phase, mb * 4) != cudaSuccess || dalloc(&c->coh_rows, mb * 4) != cudaSuccess ||
        dalloc(&c->coh_rowoff, (size_t)c->M_max * 8) != cudaSuccess)
      return fail(c, UNO_ERR_OOM, "cohort buffers");
    CK(cudaMemsetAsync(c->coh_phase, 0, mb * 4, c->stream));
    CK(cudaMemsetAsync(c->coh_drafts, 0, mb * B * 4, c->stream));
  }
  return run_graphed(
      c, 2, n_draft * 65536 + n_verify, draft_ids_dev, verify_ids_dev, out_tokens_dev,
      [&] { return cohort_step_body(c, n_draft, draft_ids_dev, n_verify, verify_ids_dev,
                                    out_tokens_dev, n_new_dev); },
      n_new_dev);
}

int uno_ar_step(uno_ctx* c, int n_req, const int32_t* req_ids_dev, int32_t* out_tokens_dev) {
  if (!c) return UNO_ERR_ARG;
  c->err.clear();
  if (n_req < 1 || n_req > c->max_batch || !req_ids_dev || !out_tokens_dev)
    return fail(c, UNO_ERR_ARG, "bad ar_step arguments");
  c->last_n_req = n_req;
  return run_graphed(c, 1, n_req, req_ids_dev, out_tokens_dev, nullptr,
                     [&] { return ar_step_body(c, n_req, req_ids_dev, out_tokens_dev); });
}

}  // extern "C"

namespace {
// Drops every captured graph: a setting baked into the kernels' arguments
// changed, so the next calls capture again.
void drop_graphs(uno_ctx* c) {
  for (auto& g : c->graphs) {
    if (g.exec) cudaGraphExecDestroy(g.exec);
    g.exec = nullptr;
    g.seen = 0;
  }
}
}  // namespace

extern "C" {

int uno_debug_set_fixed_accept(uno_ctx* c, int a) {
  if (!c) return UNO_ERR_ARG;
  if (a > c->B) return fail(c, UNO_ERR_ARG, "fixed accept beyond the block size");
  c->fixed_accept = a > 0 ? a : -1;
  drop_graphs(c);
  return UNO_OK;
}

int uno_debug_set_dep_wait(uno_ctx* c, uint64_t limit_ns, uint32_t extra) {
  if (!c || limit_ns == 0) return UNO_ERR_ARG;
  c->dep_limit_ns = limit_ns;
  c->dep_extra = extra;
  drop_graphs(c);
  return UNO_OK;
}

int uno_set_tree(uno_ctx* c, int k) {
  if (!c) return UNO_ERR_ARG;
  if (k < 1 || k > TREE_MAX_K) return fail(c, UNO_ERR_ARG, "tree chains must be in [1, 4]");
  if (k == c->tree_k) return UNO_OK;
  CK(cudaStreamSynchronize(c->stream));
  // give back the scratch pages of the previous setting
  for (int32_t pg : c->h_tree_pages) c->free_pages.push_back(pg);
  c->h_tree_pages.clear();
  c->tree_k = 1;
  drop_graphs(c);
  if (k == 1) return UNO_OK;
  const size_t mb = c->max_batch, B = c->B, V = c->s.vocab;
  if (c->free_pages.size() < 2 * (size_t)k * mb)
    return fail(c, UNO_ERR_CAPACITY, "the tree sampler needs 2 k free KV pages per request slot");
  if ((size_t)k > c->tree_cap_k) {
    void* bufs[] = {c->logits_t, c->lse_t, c->tree_chains};
    for (void* b : bufs)
      if (b) cudaFree(b);
    c->logits_t = nullptr; c->lse_t = nullptr; c->tree_chains = nullptr;
    c->tree_cap_k = 0;
    if (dalloc(&c->logits_t, mb * k * B * V * 4) != cudaSuccess ||
        dalloc(&c->lse_t, mb * k * B * 4) != cudaSuccess ||
        dalloc(&c->tree_chains, mb * k * B * 4) != cudaSuccess)
      return fail(c, UNO_ERR_OOM, "tree buffers");
    c->tree_cap_k = k;
  }
  if (!c->tree_resid) {
    if (dalloc(&c->tree_resid, mb * 2 * V * 4) != cudaSuccess ||
        dalloc(&c->tree_walk, mb * 3 * 4) != cudaSuccess ||
        dalloc(&c->tree_pages, mb * TREE_MAX_K * 2 * 4) != cudaSuccess)
      return fail(c, UNO_ERR_OOM, "tree buffers");
  }
  std::vector<int32_t> pages(mb * TREE_MAX_K * 2, 0);
  for (size_t r = 0; r < mb; ++r)
    for (int j = 0; j < k; ++j)
      for (int e = 0; e < 2; ++e) {
        const int32_t pg = c->free_pages.back();
        c->free_pages.pop_back();
        c->h_tree_pages.push_back(pg);
        pages[(r * TREE_MAX_K + j) * 2 + e] = pg;
      }
  CK(cudaMemcpy(c->tree_pages, pages.data(), pages.size() * 4, cudaMemcpyHostToDevice));
  c->tree_k = k;
  return UNO_OK;
}

int uno_set_top_p(uno_ctx* c, float top_p) {
  if (!c) return UNO_ERR_ARG;
  if (!(top_p > 0.f && top_p <= 1.f)) return fail(c, UNO_ERR_ARG, "top_p must be in (0, 1]");
  c->top_p = top_p;
  drop_graphs(c);
  return UNO_OK;
}

int uno_set_graphs(uno_ctx* c, int enable) {
  if (!c) return UNO_ERR_ARG;
  c->graphs_enabled = enable != 0;
  return UNO_OK;
}

int uno_set_counter_sync(uno_ctx* c, int enable) {
  if (!c) return UNO_ERR_ARG;
  c->counter_sync = enable != 0;
  drop_graphs(c);
  return UNO_OK;
}

int uno_set_pdl(uno_ctx* c, int enable) {
  if (!c) return UNO_ERR_ARG;
  c->genv.pdl = enable != 0;
  drop_graphs(c);   // graphs captured with the other launch mode
  return UNO_OK;
}

int uno_set_fused(uno_ctx* c, int enable) {
  if (!c) return UNO_ERR_ARG;
  c->fused_enabled = enable != 0;
  drop_graphs(c);   // graphs captured with the other pipeline
  return c->fused ? UNO_OK : UNO_ERR_UNSUPPORTED;
}

int uno_set_verify_split(uno_ctx* c, int max_ctas) {
  if (!c || max_ctas < 0) return UNO_ERR_ARG;
  c->verify_split_ctas = max_ctas;
  drop_graphs(c);
  return UNO_OK;
}

int uno_profile_records(uno_ctx* c, uno_prof_record* out, int max) {
  if (!c) return -UNO_ERR_ARG;
  const int n = (int)c->prof_done.size();
  if (out)
    for (int i = 0; i < n && i < max; ++i) out[i] = c->prof_done[i];
  return n;
}

int uno_profile_begin(uno_ctx* c, unsigned mask) {
  if (!c) return UNO_ERR_ARG;
  CK(cudaStreamSynchronize(c->stream));
  c->prof_mask = mask;
  c->prof_recs.clear();
  c->ev_next = 0;
  for (int k = 0; k < UNO_K_N; ++k) {
    c->prof_launches[k] = 0;
    c->prof_bytes[k] = 0.0;
  }
  return UNO_OK;
}

int uno_profile_end(uno_ctx* c, int64_t* launches, double* ms, double* bytes) {
  if (!c) return UNO_ERR_ARG;
  CK(cudaStreamSynchronize(c->stream));
  double t[UNO_K_N] = {};
  c->prof_done.clear();
  for (const auto& r : c->prof_recs) {
    float e = 0.f;
    CK(cudaEventElapsedTime(&e, r.a, r.b));
    t[r.cls] += e;
    c->prof_done.push_back(uno_prof_record{r.cls, r.m, r.n, r.k, r.r, e});
  }
  for (int k = 0; k < UNO_K_N; ++k) {
    if (launches) launches[k] = c->prof_launches[k];
    if (ms) ms[k] = t[k];
    if (bytes) bytes[k] = c->prof_bytes[k];
  }
  c->prof_mask = 0;
  c->prof_recs.clear();
  c->ev_next = 0;
  return UNO_OK;
}

int uno_release(uno_ctx* c, int req) {
  if (!c) return UNO_ERR_ARG;
  if (req < 0 || req >= c->max_batch || !c->slot_used[req]) return fail(c, UNO_ERR_ARG, "unknown request id");
  CK(cudaStreamSynchronize(c->stream));
  const int ppr = c->kv.pages_per_req;
  for (int pi = 0; pi < ppr; ++pi) c->free_pages.push_back(c->h_page_table[(size_t)req * ppr + pi]);
  c->slot_used[req] = 0;
  return UNO_OK;
}

int uno_status(uno_ctx* c) {
  if (!c) return UNO_ERR_ARG;
  CK(cudaStreamSynchronize(c->stream));
  int32_t st = 0;
  CK(cudaMemcpy(&st, c->d_status, 4, cudaMemcpyDeviceToHost));
  if (st) {
    CK(cudaMemset(c->d_status, 0, 4));
    return fail(c, UNO_ERR_DEVICE_CHECK, "device check flag " + std::to_string(st));
  }
  return UNO_OK;
}

int uno_request_state(uno_ctx* c, int req, int32_t* cached_out, int32_t* pending_out) {
  if (!c || !cached_out || !pending_out) return UNO_ERR_ARG;
  if (req < 0 || req >= c->max_batch || !c->slot_used[req]) return fail(c, UNO_ERR_ARG, "unknown request id");
  CK(cudaStreamSynchronize(c->stream));
  CK(cudaMemcpy(cached_out, c->d_cached + req, 4, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(pending_out, c->d_pending + req, 4, cudaMemcpyDeviceToHost));
  return UNO_OK;
}

int uno_debug_read(uno_ctx* c, int which, void* dst, size_t bytes) {
  if (!c || !dst) return UNO_ERR_ARG;
  const size_t V = c->s.vocab, B = c->B, mb = c->max_batch;
  const void* src = nullptr;
  size_t cap = 0;
  switch (which) {
    case UNO_DBG_LOGITS_DRAFT: src = c->logits_d; cap = mb * (B + 1) * V * 4; break;
    case UNO_DBG_LOGITS_VERIFY: src = c->logits_v; cap = mb * B * V * 4; break;
    case UNO_DBG_DRAFTS: src = c->drafts; cap = mb * B * 4; break;
    case UNO_DBG_LOGITS_AR: src = c->logits_d; cap = mb * V * 4; break;
    case UNO_DBG_TOPP_DRAFT: src = c->filt_d; cap = mb * (B + 1) * sizeof(RowFilter); break;
    case UNO_DBG_TOPP_VERIFY: src = c->filt_v; cap = mb * B * sizeof(RowFilter); break;
    case UNO_DBG_COHORT_LOGITS: src = c->coh_logits; cap = c->coh_logits ? 2 * mb * (B + 1) * V * 4 : 0; break;
    case UNO_DBG_COHORT_DRAFTS: src = c->coh_drafts; cap = c->coh_drafts ? mb * B * 4 : 0; break;
    case UNO_DBG_TREE_CHAINS: src = c->tree_chains; cap = c->tree_chains ? mb * c->tree_cap_k * B * 4 : 0; break;
    case UNO_DBG_TREE_LOGITS: src = c->logits_t; cap = c->logits_t ? mb * c->tree_cap_k * B * V * 4 : 0; break;
    case UNO_DBG_TREE_WALK: src = c->tree_walk; cap = c->tree_walk ? mb * 3 * 4 : 0; break;
    default: return fail(c, UNO_ERR_ARG, "unknown debug buffer");
  }
  if (bytes > cap) return fail(c, UNO_ERR_ARG, "debug read larger than the buffer");
  CK(cudaStreamSynchronize(c->stream));
  CK(cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost));
  return UNO_OK;
}

int uno_debug_kv(uno_ctx* c, int req, int layer, int pos0, int n, void* k_host, void* v_host) {
  if (!c || !k_host || !v_host) return UNO_ERR_ARG;
  if (req < 0 || req >= c->max_batch || !c->slot_used[req] || layer < 0 ||
      layer >= c->s.n_layers || pos0 < 0 || n < 0 || pos0 + n > c->max_pos)
    return fail(c, UNO_ERR_ARG, "bad debug_kv arguments");
  CK(cudaStreamSynchronize(c->stream));
  const int Hkv = c->s.n_kv_heads, hd = c->s.head_dim, ppr = c->kv.pages_per_req;
  const size_t row = (size_t)hd * c->esz;
  for (int i = 0; i < n; ++i) {
    const int pos = pos0 + i;
    const int page = c->h_page_table[(size_t)req * ppr + pos / KV_PAGE];
    for (int h = 0; h < Hkv; ++h)
      for (int kv = 0; kv < 2; ++kv) {
        const int plane = kv ? c->kv.n_planes - 1 : 0;   // K (hi), V
        const size_t off = ((((size_t)layer * c->kv.n_pages + page) * c->kv.n_planes + plane) * Hkv + h) *
                               KV_PAGE * hd +
                           (size_t)(pos % KV_PAGE) * hd;
        char* dst = (char*)(kv ? v_host : k_host) + ((size_t)i * Hkv + h) * row;
        CK(cudaMemcpy(dst, (char*)c->kv_pool + off * c->esz, row, cudaMemcpyDeviceToHost));
      }
  }
  return UNO_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// ---------------------------------------------------------------------------
// Stand-alone gated_lora_linear.
// ---------------------------------------------------------------------------
static int device_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// Workspace: counters | partial tiles | U [max(M,256), r] | X staging [256, K]
// (X is staged so that a tensor map never describes fewer rows than a box).
static constexpr int LIN_MIN_ROWS = 256;
size_t uno_gated_lora_linear_workspace_bytes(int M, int N, int K, int r, int dtype) {
  if (M < 1 || N < 1 || K < 1 || r < 0 || (dtype != UNO_F32 && dtype != UNO_BF16)) return 0;
  const size_t esz = dtype == UNO_BF16 ? 2 : 4;
  return align256((size_t)TC_COUNTERS * 4) + align256(GemmEnv::ws_bytes(device_sms())) +
         align256((size_t)std::max(M, LIN_MIN_ROWS) * std::max(r, 1) * esz) +
         align256((size_t)LIN_MIN_ROWS * K * esz);
}

int uno_debug_launch_counts(int64_t* out) {
  if (!out) return UNO_ERR_ARG;
  for (int i = 0; i < 4; ++i) out[i] = g_launches[i];
  return UNO_OK;
}

int uno_gated_lora_linear(int dtype, const void* X, const void* W, const void* A, const void* Bl,
                          const float* gate, int M, int N, int K, int r, float scale, float* Y,
                          void* ws, size_t ws_bytes, uno_stream_t stream) {
  if (!X || !W || !Y || !ws || M < 1 || N < 1 || K < 1 || (A && (!Bl || r < 1)) ||
      (dtype != UNO_F32 && dtype != UNO_BF16))
    return UNO_ERR_ARG;
  const int vec = dtype == UNO_BF16 ? 8 : 4;
  if (K % vec || (A && r % vec) || ((uintptr_t)ws & 255)) return UNO_ERR_ARG;
  if (ws_bytes < uno_gated_lora_linear_workspace_bytes(M, N, K, A ? r : 0, dtype)) return UNO_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  GemmEnv env;
  env.sm_count = device_sms();
  const size_t esz = dtype == UNO_BF16 ? 2 : 4;
  char* base = (char*)ws;
  env.counters = (unsigned*)base;
  env.ws = (float*)(base + align256((size_t)TC_COUNTERS * 4));
  void* U = base + align256((size_t)TC_COUNTERS * 4) + align256(GemmEnv::ws_bytes(env.sm_count));
  void* Xs = (char*)U + align256((size_t)std::max(M, LIN_MIN_ROWS) * std::max(A ? r : 0, 1) * esz);
  env.x_rows_alloc = std::max(M, LIN_MIN_ROWS);
  if (M < LIN_MIN_ROWS) {
    if (cudaMemcpyAsync(Xs, X, (size_t)M * K * esz, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return UNO_ERR_CUDA;
    X = Xs;
  }
  if (A) {
    GemmParams pa{};
    pa.X = X; pa.ldx = K; pa.M = M; pa.K = K; pa.N = r;
    pa.seg[0] = GemmSeg{A, nullptr, 0, r, 0};
    pa.nseg = 1;
    pa.epi = gate ? EPI_GATED : EPI_STORE;
    pa.out = U; pa.ldo = r; pa.alpha = scale; pa.row_gate = gate;
    if (dtype == UNO_BF16) gemm_run<bf16>(env, pa, st);
    else gemm_run<float>(env, pa, st);
  }
  GemmParams p{};
  p.X = X; p.ldx = K; p.M = M; p.K = K; p.N = N;
  p.seg[0] = GemmSeg{W, A ? Bl : nullptr, 0, N, 0};
  p.nseg = 1;
  if (A) { p.U = U; p.ldu = r; p.r = r; }
  p.epi = EPI_STORE_F32; p.out = Y; p.ldo = N; p.alpha = 1.f;
  if (dtype == UNO_BF16) gemm_run<bf16>(env, p, st);
  else gemm_run<float>(env, p, st);
  return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Stand-alone nucleus threshold.
// ---------------------------------------------------------------------------
int uno_top_p_filter(const float* logits, int rows, int vocab, float top_p, int32_t* out,
                     uno_stream_t stream) {
  if (!logits || !out || rows < 1 || rows > (1 << 30) || vocab < 4 || vocab % 4 ||
      ((uintptr_t)logits & 15) || !(top_p > 0.f && top_p < 1.f))
    return UNO_ERR_ARG;
  TopPArgs t{};
  t.logits = logits; t.V = vocab; t.rows_per_req = 1; t.logit_rows_per_req = 1;
  t.draft_map = 0; t.top_p = top_p; t.out = reinterpret_cast<RowFilter*>(out);
  if (!launch_top_p(false, (cudaStream_t)stream, t, rows)) return UNO_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Stand-alone spec_verify.
// ---------------------------------------------------------------------------

struct VerifyWs {
  size_t counters, req_counters, resid_counters, lse, partial, at, resid, total;
};
static VerifyWs verify_ws_layout(int n_req, int n_tests, int vocab) {
  int ch, nch;
  chunking(vocab, &ch, &nch);
  const size_t rows = (size_t)n_req * 2 * n_tests;
  VerifyWs w{};
  w.counters = 0;
  w.req_counters = align256(rows * 4);
  w.resid_counters = w.req_counters + align256((size_t)n_req * 4);
  w.lse = w.resid_counters + align256((size_t)n_req * 4);   // counters end here
  w.partial = w.lse + align256(rows * 4);
  w.at = w.partial + align256(rows * nch * sizeof(float2));
  w.resid = w.at + align256((size_t)n_req * 4);
  w.total = w.resid + align256((size_t)n_req * nch * 4);
  return w;
}

size_t uno_spec_verify_workspace_bytes(int n_req, int n_tests, int vocab) {
  if (n_req < 1 || n_tests < 1 || vocab < 4) return 0;
  return verify_ws_layout(n_req, n_tests, vocab).total;
}

// Host-side checks of a stand-alone spec_verify call (everything but the
// workspace): UNO_OK or UNO_ERR_ARG, decided before anything is enqueued.
static int verify_args_check(const float* p, const float* q, const int32_t* drafts, int n_req,
                             int n_tests, int vocab, const uint32_t* streams, const int32_t* pos0,
                             const int32_t* out_tokens, const int32_t* n_out) {
  if (!p || !q || !drafts || !streams || !pos0 || !out_tokens || !n_out) return UNO_ERR_ARG;
  if (n_req < 1 || n_tests < 1 || vocab < 4 || vocab % 4 || vocab > MAX_VOCAB || n_tests > 1024)
    return UNO_ERR_ARG;
  // grid rows of the reduction (row, chunk) CTAs
  if ((long long)n_req * 2 * n_tests > 65535LL) return UNO_ERR_ARG;
  return UNO_OK;
}

int uno_spec_verify(const float* p, const float* q, const int32_t* drafts, int n_req, int n_tests,
                    int vocab, uint64_t seed, const uint32_t* streams, const int32_t* pos0,
                    int32_t* out_tokens, int32_t* n_out, void* ws, size_t ws_bytes,
                    uno_stream_t stream) {
  const int rc = verify_args_check(p, q, drafts, n_req, n_tests, vocab, streams, pos0, out_tokens,
                                   n_out);
  if (rc != UNO_OK) return rc;
  if (!ws) return UNO_ERR_ARG;
  const VerifyWs w = verify_ws_layout(n_req, n_tests, vocab);
  if (ws_bytes < w.total || ((uintptr_t)ws & 255)) return UNO_ERR_ARG;
  int ch, nch;
  chunking(vocab, &ch, &nch);
  VerifyArgs a{};
  a.p = p; a.q = q;
  a.V = vocab; a.nch = nch; a.ch = ch;
  a.n_tests = n_tests;
  a.p_req_rows = n_tests; a.q_req_rows = n_tests;
  a.p_row0 = 0; a.q_row0 = 0;
  a.bonus_row = -1;
  a.drafts = drafts; a.drafts_stride = n_tests; a.drafts_off = 0;
  a.lse_q_in = nullptr;
  a.seed = seed;
  a.req_slot = nullptr;
  a.streams = streams; a.pos0 = pos0;
  a.out_tok = out_tokens; a.out_stride = n_tests + 1; a.n_out = n_out;
  char* base = (char*)ws;
  a.row_counter = (unsigned*)(base + w.counters);
  a.req_counter = (unsigned*)(base + w.req_counters);
  a.lse = (float*)(base + w.lse);
  a.partial = (float2*)(base + w.partial);
  a.at_ws = (int32_t*)(base + w.at);
  a.resid_part = (float*)(base + w.resid);
  a.resid_counter = (unsigned*)(base + w.resid_counters);
  a.rows_red = 2 * n_tests;
  a.n_p = n_tests;
  a.status = nullptr;
  a.fixed_at = -1;
  launch_verify(false, (cudaStream_t)stream, a, n_req);
  launch_resid(false, (cudaStream_t)stream, a, n_req, false);
  return cudaGetLastError() == cudaSuccess ? UNO_OK : UNO_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// spec_verify without allocation.
//
// Some callers cannot allocate device memory when they need this kernel: a
// serving process whose device memory is reserved up front by its own pool
// (where a stray cudaMalloc fails or breaks the budget), or code that must
// not trigger the implicit device synchronisation cudaMalloc/cudaFree can
// cause.  For them the scratch lives in a fixed array in this library's
// device image instead of a caller-provided workspace.
// ---------------------------------------------------------------------------
static constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)4 << 20;   // 4 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is asked
// for once per device (with that device current) and cached, together with
// the unique id of the device's current context: after a cudaDeviceReset
// the library's image is loaded again into a new context, the id changes
// and the address is looked up again.
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
static bool current_ctx_id(unsigned long long* id) {
  static CtxGetIdFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (CtxGetIdFn)f;
  }
  return fn && fn(nullptr, id) == CUDA_SUCCESS;   // null: the calling thread's current context
}

static int noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[256] = {};
  static unsigned long long ctx_id[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return UNO_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  if (!addr[dev] || !have_id || id != ctx_id[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return UNO_ERR_CUDA;
    addr[dev] = p;
    ctx_id[dev] = have_id ? id : 0;
  }
  *out = addr[dev];
  return UNO_OK;
}

size_t uno_spec_verify_noalloc_max_bytes(void) { return NOALLOC_SCRATCH_BYTES; }

int uno_spec_verify_noalloc(const float* p, const float* q, const int32_t* drafts, int n_req,
                            int n_tests, int vocab, uint64_t seed, const uint32_t* streams,
                            const int32_t* pos0, int32_t* out_tokens, int32_t* n_out,
                            uno_stream_t stream) {
  // every argument check before anything is enqueued on the shared array
  const int arc = verify_args_check(p, q, drafts, n_req, n_tests, vocab, streams, pos0, out_tokens,
                                    n_out);
  if (arc != UNO_OK) return arc;
  const size_t need = uno_spec_verify_workspace_bytes(n_req, n_tests, vocab);
  if (need == 0) return UNO_ERR_ARG;
  if (need > NOALLOC_SCRATCH_BYTES) return UNO_ERR_CAPACITY;
  void* ws = nullptr;
  const int rc = noalloc_scratch(&ws);
  if (rc != UNO_OK) return rc;
  // the array keeps the previous call's contents: the completion counters
  // (the first part of the layout) must start at zero
  const VerifyWs w = verify_ws_layout(n_req, n_tests, vocab);
  if (cudaMemsetAsync(ws, 0, w.lse, (cudaStream_t)stream) != cudaSuccess) return UNO_ERR_CUDA;
  return uno_spec_verify(p, q, drafts, n_req, n_tests, vocab, seed, streams, pos0, out_tokens,
                         n_out, ws, need, stream);
}

}  // extern "C"
