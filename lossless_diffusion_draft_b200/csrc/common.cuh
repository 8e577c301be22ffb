// Common device helpers of libuno: element types, Philox4x32-10 uniforms,
// warp/block reductions and the device-side error flag.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace uno {

// ---------------------------------------------------------------------------
// Element types.  Activations and weights are either fp32 or bf16; all math
// is fp32.
// ---------------------------------------------------------------------------
typedef __nv_bfloat16 bf16;
typedef __half f16;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(f16 x) { return __half2float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ f16 from_f<f16>(float x) { return __float2half_rn(x); }

// Element type of the attention operands - the rotated q rows, the paged KV
// cache and the probabilities P - for a model of element type T: fp16 for
// bf16 models (the same two bytes with three more mantissa bits; q, K, V and
// P are rounded once each), T otherwise.
template <typename T> struct KvOf { typedef T type; };
template <> struct KvOf<bf16> { typedef f16 type; };

// 16-byte vector load of VEC elements converted to fp32.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
};
template <> struct Vec16<bf16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const bf16* p, float* out) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x; out[2 * i + 1] = f.y;
    }
  }
};

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC'11).  Each round multiplies counter words 0 and 2 by
// two fixed multipliers and mixes the 64-bit products' halves with the other
// words and the key; the key advances by two Weyl constants between rounds.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k.x += 0x9E3779B9u; k.y += 0xBB67AE85u; }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
  }
  return c;
}

// Draw kinds of the sampler's uniforms.
enum DrawKind : uint32_t { KIND_FIRST = 0, KIND_DRAFT = 1, KIND_ACCEPT = 2, KIND_RESID = 3 };

// Uniform of draw `kind` for the token at absolute `pos` of random stream
// `stream`: counter (stream, pos, kind, lane), key (seed lo, seed hi), output
// word 0 mapped to ((x >> 9) * 2 + 1) * 2^-24, exact in fp32 and in (0, 1).
// lane is 0 for every draw of the linear sampler; the tree sampler numbers
// its drafted chains with it (chain 0 draws the linear sampler's uniforms).
__device__ __forceinline__ float philox_uniform(uint64_t seed, uint32_t stream, uint32_t pos,
                                                uint32_t kind, uint32_t lane = 0u) {
  const uint4 r = philox4x32_10(make_uint4(stream, pos, kind, lane),
                                make_uint2((uint32_t)seed, (uint32_t)(seed >> 32)));
  return (float)((r.x >> 9) * 2u + 1u) * (1.0f / 16777216.0f);
}

// ---------------------------------------------------------------------------
// Reductions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum / max; `red` is >= 32 floats of shared memory.  Every thread
// returns the result.  The combination order is fixed (deterministic).
template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (l < NT / 32) ? red[l] : 0.f;
  t = warp_sum(t);
  return t;
}
template <int NT>
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (l < NT / 32) ? red[l] : -INFINITY;
  t = warp_max(t);
  return t;
}

// Programmatic dependent launch.  Kernels are launched so that the next
// kernel in the stream may start while this one runs: pdl_trigger() lets it
// launch, and pdl_wait() blocks until the previous kernel has completed and
// its writes are visible.  Everything before pdl_wait() may touch only data
// no earlier kernel writes (weights, descriptors, shared memory, TMEM).
// Without a programmatic launch both return at once.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Completion counters: a finer dependency than pdl_wait() for a kernel that
// needs only the outputs of the kernel right before it.  Every CTA of the
// producer ends with dep_signal (a CTA barrier, then one release add at GPU
// scope: the CTA's writes are visible to whoever acquires the count); the
// consumer polls with acquire loads until all producer CTAs have counted.
// A consumer launched programmatically starts only after every producer CTA
// has started, so the producers it waits for are all resident and the wait
// ends; it is bounded anyway (false after about a second).  The counters of
// a pass are zeroed by its first kernel after that kernel's pdl_wait() and
// before its pdl_trigger(), so no kernel of the pass can see a stale count.
__device__ __forceinline__ void dep_signal(unsigned* ctr) {   // whole CTA, at its end
  if (!ctr) return;
  __syncthreads();
  if (threadIdx.x == 0 && threadIdx.y == 0)
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}
// The same for a CTA that has just passed a barrier after its last write.
__device__ __forceinline__ void dep_signal_synced(unsigned* ctr) {
  if (ctr && threadIdx.x == 0 && threadIdx.y == 0)
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}
// limit_ns: how long to poll (global timer) before giving up.
__device__ __forceinline__ bool dep_wait(const unsigned* ctr, unsigned target,
                                         unsigned long long limit_ns) {   // one thread
  unsigned long long t0 = 0;
  for (int i = 0;; ++i) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (i == 0) t0 = t;
    else if (t - t0 > limit_ns) return false;
    __nanosleep(20);
  }
}

// Device-side error flag bits (read by uno_status).
enum StatusBits : int32_t {
  ST_POS_OVERFLOW = 1,   // a position beyond the request's KV pages
  ST_BAD_TOKEN = 2,      // a token id outside [0, vocab)
  ST_BAD_SLOT = 4,       // a request id outside [0, max_batch) or not admitted
  ST_DEP_TIMEOUT = 32,   // a completion-counter wait gave up
};
__device__ __forceinline__ void raise_status(int32_t* st, int32_t bit) {
  if (st) atomicOr(st, bit);
}

}  // namespace uno
