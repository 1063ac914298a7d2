// Loop-axis VQ encode (sm_100a): nearest codeword in squared L2.
//
// LoopVQ project page, "Method" -- "Overview of LoopVQ" and "Component 1":
// the sub-vector of (code block b, head h, slot j, token n) gathers channels
// j*W .. j*W+W-1 of the Tc consecutive loop steps b*Tc .. b*Tc+Tc-1, and one
// codebook index replaces it.  Distances are sum_g (x_g - c_g)^2 in fp32,
// taken from the differences (no norm expansion, so no cancellation near a
// match); the scan runs over c = 0, 1, ... with a strict "<", so ties go to
// the lowest index.
//
// Work split: one CTA per (slot j, token chunk, code block b x head h) with
// j fastest, so the CTAs that share a token chunk run together and reuse its
// sectors in L2.  The (b, h, j) codebook (C x G fp32) sits in shared memory
// and is read by broadcast; each thread holds TPT sub-vectors in registers.

#include "common.cuh"

namespace loopvq {

struct EncodeParams {
  const void* x;
  int x_bf16;
  int64_t st, sn, sh;  // element strides of t, n, h
  int64_t n_tokens;
  const void* cb;      // canonical [NB][H][J][C][Tc][W]
  int cb_bf16;
  int Tc, H, J, W, C, kind;
  uint8_t* pool;
  int64_t tok_off, pool_tokens;
};

template <int G, int TPT>
__global__ void __launch_bounds__(256) encode_kernel(const EncodeParams p) {
  extern __shared__ __align__(16) float cbs[];  // [C][G]
  const int j = blockIdx.x;
  const int bh = blockIdx.z;
  const int b = bh / p.H, h = bh % p.H;
  const int64_t cb_off = ((int64_t)bh * p.J + j) * p.C * G;
  for (int e = threadIdx.x; e < p.C * G; e += blockDim.x)
    cbs[e] = p.cb_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.cb)[cb_off + e])
                       : reinterpret_cast<const float*>(p.cb)[cb_off + e];
  __syncthreads();

  const int64_t n_base = (int64_t)blockIdx.y * (256 * TPT) + threadIdx.x;
  float x[TPT][G];
#pragma unroll
  for (int k = 0; k < TPT; ++k) {
    const int64_t n = n_base + 256 * k;
    const bool ok = n < p.n_tokens;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      // element (tt, w) of the sub-vector sits at g = tt*W + w
      const int tt = g / p.W, w = g - tt * p.W;
      float v = 0.f;
      if (ok) {
        const int64_t e = (int64_t)(b * p.Tc + tt) * p.st + n * p.sn + (int64_t)h * p.sh + (int64_t)j * p.W + w;
        v = p.x_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.x)[e])
                     : reinterpret_cast<const float*>(p.x)[e];
      }
      x[k][g] = v;
    }
  }

  float best[TPT];
  int bi[TPT];
#pragma unroll
  for (int k = 0; k < TPT; ++k) { best[k] = INFINITY; bi[k] = 0; }
  for (int c = 0; c < p.C; ++c) {
    const float* row = cbs + c * G;
    float cv[G];
#pragma unroll
    for (int g = 0; g < G; g += 4) {
      if constexpr (G % 4 == 0) {
        float4 t4 = *reinterpret_cast<const float4*>(row + g);
        cv[g] = t4.x; cv[g + 1] = t4.y; cv[g + 2] = t4.z; cv[g + 3] = t4.w;
      } else {
        for (int q = g; q < G && q < g + 4; ++q) cv[q] = row[q];
      }
    }
#pragma unroll
    for (int k = 0; k < TPT; ++k) {
      float d = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float df = x[k][g] - cv[g];
        d = fmaf(df, df, d);
      }
      if (d < best[k]) { best[k] = d; bi[k] = c; }
    }
  }
#pragma unroll
  for (int k = 0; k < TPT; ++k) {
    const int64_t n = n_base + 256 * k;
    if (n < p.n_tokens)
      p.pool[pool_byte(p.J, p.kind, p.pool_tokens, b, p.H, h, p.tok_off + n, j)] = (uint8_t)bi[k];
  }
}

// Few-token encode (a page of the recent window, a short prompt): one CTA per
// (slot j, chunk of kSmallTok tokens, b x h); the codebook is staged in shared
// memory transposed to [G][C] so that lane l reading codes l, l+32, ... hits
// 32 different banks.  Each warp takes one token at a time: every lane scans
// its C/32 codes in increasing order with the same fp32 arithmetic as above,
// then the warp picks the smallest (distance, code) pair -- the same code as
// the sequential scan, ties to the lowest index.
constexpr int kSmallTok = 64;
constexpr int kSmallWarps = 8;

template <int G>
__global__ void __launch_bounds__(kSmallWarps * 32) encode_small_kernel(const EncodeParams p) {
  extern __shared__ __align__(16) float cbt[];  // [G][C]
  const int j = blockIdx.x;
  const int bh = blockIdx.z;
  const int b = bh / p.H, h = bh % p.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t cb_off = ((int64_t)bh * p.J + j) * p.C * G;
  // thread c loads codeword c whole (one round of load latency) and spreads
  // it over column c of the [G][C] table (consecutive c: distinct banks)
  for (int c = threadIdx.x; c < p.C; c += blockDim.x) {
    float v[G];
    if (p.cb_bf16) {
      const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(p.cb) + cb_off + (int64_t)c * G;
      if constexpr (G % 8 == 0) {
#pragma unroll
        for (int k = 0; k < G / 8; ++k) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(src) + k);
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) { v[8 * k + 2 * i] = bf16_lo(w[i]); v[8 * k + 2 * i + 1] = bf16_hi(w[i]); }
        }
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) v[g] = __bfloat162float(__ldg(src + g));
      }
    } else {
      const float* src = reinterpret_cast<const float*>(p.cb) + cb_off + (int64_t)c * G;
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int k = 0; k < G / 4; ++k) {
          const float4 u = __ldg(reinterpret_cast<const float4*>(src) + k);
          v[4 * k] = u.x; v[4 * k + 1] = u.y; v[4 * k + 2] = u.z; v[4 * k + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) v[g] = __ldg(src + g);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) cbt[g * p.C + c] = v[g];
  }
  __syncthreads();
  const int64_t n0 = (int64_t)blockIdx.y * kSmallTok;
  for (int k = warp; k < kSmallTok; k += kSmallWarps) {
    const int64_t n = n0 + k;
    if (n >= p.n_tokens) break;  // warp-uniform
    float x[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int tt = g / p.W, w = g - tt * p.W;
      const int64_t e = (int64_t)(b * p.Tc + tt) * p.st + n * p.sn + (int64_t)h * p.sh + (int64_t)j * p.W + w;
      x[g] = p.x_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.x)[e])
                      : reinterpret_cast<const float*>(p.x)[e];
    }
    float best = INFINITY;
    int bi = 0x7FFFFFFF;
    for (int c = lane; c < p.C; c += 32) {
      float d = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float df = x[g] - cbt[g * p.C + c];
        d = fmaf(df, df, d);
      }
      if (d < best) { best = d; bi = c; }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob < best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    if (lane == 0) p.pool[pool_byte(p.J, p.kind, p.pool_tokens, b, p.H, h, p.tok_off + n, j)] = (uint8_t)bi;
  }
}

bool encode_tc_try(const Geo& g, const void* cb, int kind, const void* x, int64_t n_tokens, int64_t st, int64_t sn,
                   int64_t sh, uint8_t* pool, int64_t tok_off, int64_t pool_tokens, uint32_t* faults, cudaStream_t s,
                   cudaError_t* err);

// Below this many tokens a 128-row tensor-core tile or a 256-thread chunk is
// mostly padding, and the few-token kernel runs instead.
constexpr int64_t kSmallMaxTokens = 256;

}  // namespace loopvq

using namespace loopvq;

extern "C" loopvq_status loopvq_encode(const loopvq_codebook_desc* desc, const void* cb_packed, loopvq_kind kind,
                                       const void* x, loopvq_dtype x_dtype, int64_t n_tokens, int64_t stride_t,
                                       int64_t stride_n, int64_t stride_h, uint8_t* idx_pool, int64_t tok_off,
                                       int64_t pool_tokens, uint32_t* fault_bits, loopvq_stream_t stream) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if (kind != LOOPVQ_KEYS && kind != LOOPVQ_VALUES) return LOOPVQ_ERR_INVALID_ARG;
  if (x_dtype != LOOPVQ_F32 && x_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens < 0 || tok_off < 0 || pool_tokens <= 0 || (pool_tokens & 31) || tok_off + n_tokens > pool_tokens)
    return LOOPVQ_ERR_INVALID_ARG;
  if (stride_t < 0 || stride_n < 0 || stride_h < 0) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens == 0) return LOOPVQ_OK;
  if (!cb_packed || !x || !idx_pool || ((uintptr_t)cb_packed & 15) || ((uintptr_t)fault_bits & 3))
    return LOOPVQ_ERR_INVALID_ARG;

  EncodeParams p;
  p.x = x; p.x_bf16 = x_dtype == LOOPVQ_BF16;
  p.st = stride_t; p.sn = stride_n; p.sh = stride_h;
  p.n_tokens = n_tokens;
  p.cb = cb_packed; p.cb_bf16 = g.cb_bf16;
  p.Tc = g.Tc; p.H = g.H; p.J = g.J; p.W = g.W; p.C = g.C; p.kind = (int)kind;
  p.pool = idx_pool; p.tok_off = tok_off; p.pool_tokens = pool_tokens;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t smem = (size_t)g.C * g.G * sizeof(float);
  if ((int64_t)g.NB * g.H > 65535) return LOOPVQ_ERR_UNSUPPORTED;
  if (n_tokens < kSmallMaxTokens) {
    const int64_t chunks = (n_tokens + kSmallTok - 1) / kSmallTok;
    dim3 grid(g.J, (unsigned)chunks, g.NB * g.H);
#define LOOPVQ_SMALL(GG)                                                                                   \
  do {                                                                                                    \
    if (smem > 48 * 1024 && cudaFuncSetAttribute(encode_small_kernel<GG>,                                 \
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != \
                                cudaSuccess)                                                              \
      return LOOPVQ_ERR_CUDA;                                                                             \
    encode_small_kernel<GG><<<grid, kSmallWarps * 32, smem, s>>>(p);                                      \
  } while (0)
    switch (g.G) {
      case 2: LOOPVQ_SMALL(2); break;
      case 4: LOOPVQ_SMALL(4); break;
      case 8: LOOPVQ_SMALL(8); break;
      case 16: LOOPVQ_SMALL(16); break;
      case 32: LOOPVQ_SMALL(32); break;
      case 64: LOOPVQ_SMALL(64); break;
      default: return LOOPVQ_ERR_UNSUPPORTED;
    }
#undef LOOPVQ_SMALL
    return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
  }
  if (p.x_bf16) {
    cudaError_t e = cudaSuccess;
    if (encode_tc_try(g, cb_packed, (int)kind, x, n_tokens, stride_t, stride_n, stride_h, idx_pool, tok_off,
                      pool_tokens, fault_bits, s, &e))
      return e == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
  }
#define LOOPVQ_ENC(GG, TT)                                                                       \
  do {                                                                                          \
    const int64_t chunks = (n_tokens + 256 * TT - 1) / (256 * TT);                              \
    if (chunks > 65535) return LOOPVQ_ERR_UNSUPPORTED;                                          \
    dim3 grid(g.J, (unsigned)chunks, g.NB * g.H);                                               \
    if (smem > 48 * 1024 &&                                                                     \
        cudaFuncSetAttribute(encode_kernel<GG, TT>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)smem) != cudaSuccess)                                         \
      return LOOPVQ_ERR_CUDA;                                                                   \
    encode_kernel<GG, TT><<<grid, 256, smem, s>>>(p);                                           \
  } while (0)
  switch (g.G) {
    case 2: LOOPVQ_ENC(2, 8); break;
    case 4: LOOPVQ_ENC(4, 8); break;
    case 8: LOOPVQ_ENC(8, 8); break;
    case 16: LOOPVQ_ENC(16, 4); break;
    case 32: LOOPVQ_ENC(32, 2); break;
    case 64: LOOPVQ_ENC(64, 1); break;
    default: return LOOPVQ_ERR_UNSUPPORTED;
  }
#undef LOOPVQ_ENC
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}
