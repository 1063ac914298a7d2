// Internal helpers shared by the libloopvq translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "loopvq.h"

namespace loopvq {

// ---------------------------------------------------------------- geometry
// Derived sizes of a descriptor (LoopVQ project page, "Overview of LoopVQ":
// a code spans W = G/Tc channels of each of Tc loop steps; J = D/W slots).
struct Geo {
  int T, Tc, NB, H, Hq, D, G, W, J, C;
  bool cb_bf16;
};

// Returns LOOPVQ_OK and fills g, or the validation status.
loopvq_status make_geo(const loopvq_codebook_desc* d, Geo* g);

inline size_t cb_elem_bytes(const Geo& g) { return g.cb_bf16 ? 2 : 4; }
inline size_t canonical_elems(const Geo& g) { return (size_t)g.NB * g.H * g.J * g.C * g.Tc * g.W; }
// Per-step slices [T][H][C][J][W] follow the canonical block in the packed form.
inline size_t slice_elems_per_step(const Geo& g) { return (size_t)g.H * g.C * g.J * g.W; }
inline size_t packed_slices_offset_bytes(const Geo& g) {
  size_t b = canonical_elems(g) * cb_elem_bytes(g);
  return (b + 255) & ~(size_t)255;
}

// ------------------------------------------------------------ pool layout
// A pool stream is [NB][H][pool_tokens/32][tile]; a tile holds 32 tokens x J
// slots, one uint8 code each.  Token n of a tile is read by lane n of a warp
// in 16-byte pieces (one piece for J <= 16, two for J = 32): piece p of token
// n sits at p*512 + n*min(J,16), so each warp-wide piece load is one
// contiguous 512-byte (or 256-byte) run.  Inside a token's J bytes the codes
// are rotated: byte s holds slot (s + n) mod J.  At step s of the decode loops
// the 32 lanes therefore touch 32 different slots, i.e. 32 different shared
// memory banks of the per-slot lookup tables and histograms.  K and V tiles
// use the same order.
__host__ __device__ inline int64_t tile_byte(int J, int kind, int n_in_tile, int j) {
  (void)kind;
  const int s = ((j - n_in_tile) % J + J) % J;
  const int piece = J < 16 ? J : 16;
  return (int64_t)(s / piece) * (32 * piece) + (int64_t)n_in_tile * piece + (s % piece);
}
__host__ __device__ inline int64_t pool_byte(int J, int kind, int64_t pool_tokens, int b, int H, int h,
                                             int64_t n, int j) {
  int64_t tile = n >> 5;
  int64_t stream = (int64_t)b * H + h;
  return (stream * (pool_tokens >> 5) + tile) * (32LL * J) + tile_byte(J, kind, (int)(n & 31), j);
}

// ------------------------------------------------------- workspace layout
// [0, 256)            status word (u32 at 0)
// [256, 256+tickets)  u32 split counters, one per (request, query head)
// then                fp32 partials [units][max_splits][D + 4]: o[D], m, l, pad
struct WsLayout {
  size_t tickets_off, partials_off, total;
};
inline WsLayout ws_layout(int64_t units, int max_splits, int D) {
  WsLayout w;
  w.tickets_off = 256;
  size_t tb = (size_t)units * 4;
  w.partials_off = (w.tickets_off + tb + 255) & ~(size_t)255;
  w.total = w.partials_off + (size_t)units * max_splits * (D + 4) * sizeof(float);
  return w;
}

// ------------------------------------------------------ window split rule
// Project page, "Serving in SGLang": first n_sink and most recent n_recent
// tokens bf16; pages of `page` tokens are encoded once the recent window has
// a full extra page, so the recent window holds n_recent + ((ctx - n_sink -
// n_recent) mod page) tokens.  A context within n_sink + n_recent is all bf16.
struct CtxSplit { int sink, body, recent; };
__host__ __device__ inline CtxSplit ctx_split(int ctx, int n_sink, int n_recent, int page) {
  CtxSplit s;
  if (ctx <= n_sink + n_recent) {
    s.sink = ctx < n_sink ? ctx : n_sink;
    s.body = 0;
    s.recent = ctx - s.sink;
  } else {
    int extra = (ctx - n_sink - n_recent) % page;
    s.sink = n_sink;
    s.recent = n_recent + extra;
    s.body = ctx - n_sink - s.recent;
  }
  return s;
}

// Number of SMs of the current device (148 on B200); falls back to 148.
int device_sm_count();

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false after ~`limit` polls (each poll already blocks
// for a hardware-defined slice), so a lost completion can never hang the GPU.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t limit = 1u << 20) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
// TMA bulk copy global -> shared (no multicast), completion on an mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ void set_fault(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// Combine of split partials for one (request, query head): the last split to
// finish merges every split's (o[D], m, l) by log-sum-exp; m is in log2 units
// and o is unnormalised (sum of weights 2^(s - m) times values).  All loads of
// a phase are independent so they are in flight together: phase 1 stages
// every split's (m, l) in shared memory, phase 2 has nthr/D threads per
// output channel each summing a stride of the splits, phase 3 adds those up.
// `sm` holds 2*kMaxCombineSplits + nthr floats; `sync` is the CTA barrier of
// the nthr participating threads (tid in [0, nthr)).
constexpr int kMaxCombineSplits = 1024;
struct BlockSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
template <typename Sync>
__device__ __forceinline__ void combine_splits(const float* part, int n_splits, int D, void* out, int out_bf16,
                                               float* lse, float* sm, int tid, int nthr, Sync sync) {
  float* sm_m = sm;
  float* sm_l = sm + kMaxCombineSplits;
  float* sm_acc = sm + 2 * kMaxCombineSplits;
  const size_t stride = (size_t)(D + 4);
  for (int s = tid; s < n_splits; s += nthr) {
    sm_m[s] = __ldcg(part + s * stride + D);
    sm_l[s] = __ldcg(part + s * stride + D + 1);
  }
  sync();
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, sm_m[s]);
  float L = 0.f;
  for (int s = 0; s < n_splits; ++s)
    if (sm_m[s] != -INFINITY) L += sm_l[s] * exp2f(sm_m[s] - M);
  const int P = nthr / D;
  const int d = tid % D, pi = tid / D;
  float acc = 0.f;
  if (pi < P && M != -INFINITY) {
    int s = pi;
    for (; s + 3 * P < n_splits; s += 4 * P) {
      const float a0 = __ldcg(part + s * stride + d);
      const float a1 = __ldcg(part + (s + P) * stride + d);
      const float a2 = __ldcg(part + (s + 2 * P) * stride + d);
      const float a3 = __ldcg(part + (s + 3 * P) * stride + d);
      const float w0 = sm_m[s] != -INFINITY ? exp2f(sm_m[s] - M) : 0.f;
      const float w1 = sm_m[s + P] != -INFINITY ? exp2f(sm_m[s + P] - M) : 0.f;
      const float w2 = sm_m[s + 2 * P] != -INFINITY ? exp2f(sm_m[s + 2 * P] - M) : 0.f;
      const float w3 = sm_m[s + 3 * P] != -INFINITY ? exp2f(sm_m[s + 3 * P] - M) : 0.f;
      acc = fmaf(a0, w0, fmaf(a1, w1, fmaf(a2, w2, fmaf(a3, w3, acc))));
    }
    for (; s < n_splits; s += P)
      if (sm_m[s] != -INFINITY) acc = fmaf(__ldcg(part + s * stride + d), exp2f(sm_m[s] - M), acc);
  }
  if (pi < P) sm_acc[pi * D + d] = acc;
  sync();
  if (tid < D) {
    float o = 0.f;
    for (int i = 0; i < P; ++i) o += sm_acc[i * D + tid];
    o = (M != -INFINITY && L > 0.f) ? o / L : 0.f;
    if (out_bf16)
      ((__nv_bfloat16*)out)[tid] = __float2bfloat16_rn(o);
    else
      ((float*)out)[tid] = o;
  }
  if (lse && tid == 0) *lse = (M == -INFINITY || !(L > 0.f)) ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
}

}  // namespace loopvq
