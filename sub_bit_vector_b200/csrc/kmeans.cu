// Lloyd update of the loop-axis codebooks (sm_100a): codebook construction.
//
// LoopVQ project page, "Method" -- "Loop-aware codebook fine-tuning": the
// codebooks are fine-tuned against the full-precision model; the pages do not
// say where that starts.  The data-driven start is Lloyd's k-means on the
// same loop-axis sub-vectors the encoder codes: alternate loopvq_encode (the
// nearest-codeword assignment) with this update, which takes codeword c of
// (block b, head h, slot j) to the mean of the sub-vectors stored with code
// c and leaves unused codewords as they were.
//
// Two kernels.  Accumulate: one CTA per (slot j, chunk of tokens, b x h)
// sums its sub-vectors per code in shared memory ([C][G+1] fp32, the last
// column counting members; G+1 is odd, so neighbouring codes fall in
// different banks) and flushes the non-zero entries to a global fp32
// workspace with atomics.  Finalize: one thread per codebook element divides
// the sum by the count (or copies the old value) and writes the canonical
// codebook.

#include "common.cuh"

namespace loopvq {

constexpr int kKmTok = 2048;     // tokens per accumulate CTA
constexpr int kKmThreads = 256;

struct KmParams {
  const void* x;
  int x_bf16;
  int64_t st, sn, sh;
  int64_t n_tokens;
  const uint8_t* pool;
  int kind;
  int64_t tok_off, pool_tokens;
  int Tc, H, J, W, G, C;
  float* sums;       // [NB][H][J][C][G]
  float* counts;     // [NB][H][J][C]
};

__global__ void __launch_bounds__(kKmThreads) km_accumulate_kernel(const KmParams p) {
  extern __shared__ float acc[];  // [C][G + 1]
  const int j = blockIdx.x;
  const int bh = blockIdx.z;
  const int b = bh / p.H, h = bh % p.H;
  const int row = p.G + 1;
  for (int e = threadIdx.x; e < p.C * row; e += blockDim.x) acc[e] = 0.f;
  __syncthreads();
  const int64_t n0 = (int64_t)blockIdx.y * kKmTok;
  const int64_t n1 = min(p.n_tokens, n0 + kKmTok);
  for (int64_t n = n0 + threadIdx.x; n < n1; n += blockDim.x) {
    const int c = p.pool[pool_byte(p.J, p.kind, p.pool_tokens, b, p.H, h, p.tok_off + n, j)];
    if (c >= p.C) continue;  // not a code of this codebook: ignored
    float* dst = acc + c * row;
    for (int g = 0; g < p.G; ++g) {
      const int tt = g / p.W, w = g - tt * p.W;
      const int64_t e = (int64_t)(b * p.Tc + tt) * p.st + n * p.sn + (int64_t)h * p.sh + (int64_t)j * p.W + w;
      const float v = p.x_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.x)[e])
                               : reinterpret_cast<const float*>(p.x)[e];
      atomicAdd(dst + g, v);
    }
    atomicAdd(dst + p.G, 1.f);
  }
  __syncthreads();
  const size_t cbase = (((size_t)bh * p.J) + j) * p.C;
  for (int e = threadIdx.x; e < p.C * row; e += blockDim.x) {
    const float v = acc[e];
    if (v == 0.f) continue;
    const int c = e / row, g = e - c * row;
    if (g < p.G)
      atomicAdd(p.sums + (cbase + c) * p.G + g, v);
    else
      atomicAdd(p.counts + cbase + c, v);
  }
}

template <typename CBT>
__global__ void km_finalize_kernel(const float* sums, const float* counts, const CBT* cb_in, CBT* cb_out,
                                   int32_t* counts_out, int64_t n_codewords, int G) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // element of [..][C][G]
  if (e >= n_codewords * G) return;
  const int64_t cw = e / G;
  const float cnt = counts[cw];
  // canonical codeword (t, w) sits at t*W + w, the same order as the sums
  if (cnt > 0.f) {
    const float mean = sums[e] / cnt;
    if constexpr (sizeof(CBT) == 2)
      cb_out[e] = __float2bfloat16_rn(mean);
    else
      cb_out[e] = mean;
  } else {
    cb_out[e] = cb_in[e];
  }
  if (counts_out && e % G == 0) counts_out[cw] = (int32_t)cnt;
}

}  // namespace loopvq

using namespace loopvq;

extern "C" size_t loopvq_codebook_update_workspace_bytes(const loopvq_codebook_desc* desc) {
  Geo g;
  if (make_geo(desc, &g) != LOOPVQ_OK) return 0;
  const size_t cw = (size_t)g.NB * g.H * g.J * g.C;
  return cw * g.G * sizeof(float) + ((cw * sizeof(float) + 255) & ~(size_t)255) + 256;
}

extern "C" loopvq_status loopvq_codebook_update(const loopvq_codebook_desc* desc, loopvq_kind kind, const void* x,
                                                loopvq_dtype x_dtype, int64_t n_tokens, int64_t stride_t,
                                                int64_t stride_n, int64_t stride_h, const uint8_t* idx_pool,
                                                int64_t tok_off, int64_t pool_tokens, const void* cb_in,
                                                void* cb_out, int32_t* counts_out, void* workspace,
                                                size_t workspace_bytes, loopvq_stream_t stream) {
  Geo g;
  loopvq_status st = make_geo(desc, &g);
  if (st != LOOPVQ_OK) return st;
  if (kind != LOOPVQ_KEYS && kind != LOOPVQ_VALUES) return LOOPVQ_ERR_INVALID_ARG;
  if (x_dtype != LOOPVQ_F32 && x_dtype != LOOPVQ_BF16) return LOOPVQ_ERR_INVALID_ARG;
  if (n_tokens < 0 || tok_off < 0 || pool_tokens <= 0 || (pool_tokens & 31) || tok_off + n_tokens > pool_tokens)
    return LOOPVQ_ERR_INVALID_ARG;
  if (stride_t < 0 || stride_n < 0 || stride_h < 0) return LOOPVQ_ERR_INVALID_ARG;
  if (!x || !idx_pool || !cb_in || !cb_out || !workspace) return LOOPVQ_ERR_INVALID_ARG;
  if (cb_in == cb_out) return LOOPVQ_ERR_INVALID_ARG;
  if ((uintptr_t)workspace & 255) return LOOPVQ_ERR_INVALID_ARG;
  if (workspace_bytes < loopvq_codebook_update_workspace_bytes(desc)) return LOOPVQ_ERR_WORKSPACE_TOO_SMALL;
  if ((int64_t)g.NB * g.H > 65535) return LOOPVQ_ERR_UNSUPPORTED;
  const int64_t chunks = (n_tokens + kKmTok - 1) / kKmTok;
  if (chunks > 65535) return LOOPVQ_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t cw = (size_t)g.NB * g.H * g.J * g.C;
  float* sums = (float*)workspace;
  float* counts = (float*)((uint8_t*)workspace + ((cw * g.G * sizeof(float) + 255) & ~(size_t)255));
  if (cudaMemsetAsync(workspace, 0, loopvq_codebook_update_workspace_bytes(desc), s) != cudaSuccess)
    return LOOPVQ_ERR_CUDA;
  KmParams p;
  p.x = x; p.x_bf16 = x_dtype == LOOPVQ_BF16;
  p.st = stride_t; p.sn = stride_n; p.sh = stride_h;
  p.n_tokens = n_tokens;
  p.pool = idx_pool; p.kind = (int)kind; p.tok_off = tok_off; p.pool_tokens = pool_tokens;
  p.Tc = g.Tc; p.H = g.H; p.J = g.J; p.W = g.W; p.G = g.G; p.C = g.C;
  p.sums = sums; p.counts = counts;
  if (n_tokens > 0) {
    const size_t smem = (size_t)g.C * (g.G + 1) * sizeof(float);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(km_accumulate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
      return LOOPVQ_ERR_CUDA;
    dim3 grid(g.J, (unsigned)chunks, g.NB * g.H);
    km_accumulate_kernel<<<grid, kKmThreads, smem, s>>>(p);
  }
  const int64_t n_el = (int64_t)cw * g.G;
  const unsigned blocks = (unsigned)((n_el + 255) / 256);
  if (g.cb_bf16)
    km_finalize_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(sums, counts, (const __nv_bfloat16*)cb_in,
                                                             (__nv_bfloat16*)cb_out, counts_out, (int64_t)cw, g.G);
  else
    km_finalize_kernel<float><<<blocks, 256, 0, s>>>(sums, counts, (const float*)cb_in, (float*)cb_out, counts_out,
                                                     (int64_t)cw, g.G);
  return cudaGetLastError() == cudaSuccess ? LOOPVQ_OK : LOOPVQ_ERR_CUDA;
}
