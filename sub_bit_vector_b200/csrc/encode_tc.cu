// Loop-axis VQ encode on the 5th-generation tensor cores (sm_100a).
//
// LoopVQ project page, "Method" -- "Overview of LoopVQ" and "Component 1":
// each loop-axis sub-vector x (G elements: W channels of each of Tc
// consecutive loop steps) is replaced by the index of its nearest codeword.
// For bf16 inputs and 256-entry bf16 codebooks the distance block is a dense
// contraction,
//
//   d(n, c) = ||x_n||^2 + ||c||^2 - 2 x_n . c ,
//
// computed for a tile of 128 sub-vectors x 256 codewords by tcgen05.mma (bf16
// operands in shared memory, fp32 accumulator in tensor memory).  The norms
// ride in the contraction: K is padded from G to a multiple of 16 and the pad
// holds each norm split exactly into three bf16 parts (hi + mid + lo equals
// the fp32 value) against ones on the other operand, so the accumulator holds
// d itself.  Every product of two bf16 values is exact in fp32; only the sums
// round.
//
// Epilogue (one thread per sub-vector = one TMEM lane): the row's norm
// carries a small positive bias (the same for every codeword) that keeps the
// fast distances positive.  A candidate's key is its fast distance rounded to
// an integer at a per-row power-of-two scale (23 bits) with the code below
// it, so keys order like d and break ties by code.  Four chains of sorted
// key pairs keep each chain's two smallest keys; chain c covers the
// 8-column groups 32g + 8c.  When the two smallest keys of the row are
// closer than twice a bound on the fast path's error (plus the keys'
// rounding), the row is re-solved exactly, in fp32 from the differences
// sum_g (x_g - c_g)^2, ties to the lower code, over every codeword whose fast
// distance is within that bound of the minimum: the chain heads within the
// bound, plus the columns of any chain whose second key is within it (its
// third is not kept), re-read from TMEM.  The result is the nearest codeword
// except where two are within fp32 rounding of each other -- the guarantee
// of the CUDA-core encoder.

#include "common.cuh"

namespace loopvq {

constexpr int kTcTile = 128;        // sub-vectors per MMA tile (M)
constexpr int kTcCodes = 256;       // codewords (N)
constexpr int kTcThreads = 128;     // one thread per tile row
constexpr int kTcTilesPerCta = 32;  // 4096 tokens per CTA
// Shared memory asked per CTA: at most two CTAs share an SM, so their two
// 256-column accumulators fit the SM's 512 TMEM columns and tcgen05.alloc
// never has to wait for another CTA.
constexpr int kTcSmemFloor = 80 * 1024;

struct EncodeTcParams {
  const __nv_bfloat16* x;
  int64_t st, sn, sh;  // element strides of t, n, h
  int64_t n_tokens;
  const __nv_bfloat16* cb;  // canonical [NB][H][J][C][Tc][W]
  int Tc, H, J, W, kind;
  uint8_t* pool;
  int64_t tok_off, pool_tokens;
  uint32_t* faults;  // caller's fault word, or null
  // 256, passed at run time: the key's bits * 256 + code then issues as an
  // integer multiply-add (FMA pipe) instead of a shift and add on the integer
  // ALU pipe, which the top-2 min/max keep busy (measured 1.56 vs 1.65 ms)
  uint32_t key_mul;
};

// ---- canonical K-major, no-swizzle operand layout ---------------------------
// A [rows][KP] bf16 operand is stored as 8-row x 16-byte core matrices of 128
// contiguous bytes; core (r/8, k/8) sits at (r/8)*SBO + (k/8)*LBO with
// LBO = 128 B (next 8 elements of K) and SBO = KP/8 * 128 B (next 8 rows).
template <int KP>
__device__ __forceinline__ uint32_t core_off(int r, int k8) {
  return (uint32_t)((r >> 3) * (KP / 8) * 128 + k8 * 128 + (r & 7) * 16);
}
template <int KP>
__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t saddr) {
  constexpr uint64_t lbo = 128, sbo = (KP / 8) * 128;
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= ((lbo >> 4) & 0x3FFF) << 16;
  d |= ((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;  // sm_100 descriptor version; base offset 0, no swizzle
  return d;
}
// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kTcIdesc =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcCodes >> 3) << 17) | ((uint32_t)(kTcTile >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t dtmem, uint64_t ad, uint64_t bd, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(dtmem),
      "l"(ad), "l"(bd), "r"(kTcIdesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void tmem_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
// Waits for the outstanding TMEM loads and ties r to the wait, so that no use
// of the loaded registers can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld_tied(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
// Waits for the outstanding TMEM loads, tied to the 64 registers of r.
__device__ __forceinline__ void tmem_wait_ld_tied64(uint32_t (&r)[8][8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0][0]), "+r"(r[0][1]), "+r"(r[0][2]), "+r"(r[0][3]), "+r"(r[0][4]), "+r"(r[0][5]),
                 "+r"(r[0][6]), "+r"(r[0][7]), "+r"(r[1][0]), "+r"(r[1][1]), "+r"(r[1][2]), "+r"(r[1][3]),
                 "+r"(r[1][4]), "+r"(r[1][5]), "+r"(r[1][6]), "+r"(r[1][7]), "+r"(r[2][0]), "+r"(r[2][1]),
                 "+r"(r[2][2]), "+r"(r[2][3]), "+r"(r[2][4]), "+r"(r[2][5]), "+r"(r[2][6]), "+r"(r[2][7]),
                 "+r"(r[3][0]), "+r"(r[3][1]), "+r"(r[3][2]), "+r"(r[3][3]), "+r"(r[3][4]), "+r"(r[3][5]),
                 "+r"(r[3][6]), "+r"(r[3][7])
               :
               : "memory");
  asm volatile(""
               : "+r"(r[4][0]), "+r"(r[4][1]), "+r"(r[4][2]), "+r"(r[4][3]), "+r"(r[4][4]), "+r"(r[4][5]),
                 "+r"(r[4][6]), "+r"(r[4][7]), "+r"(r[5][0]), "+r"(r[5][1]), "+r"(r[5][2]), "+r"(r[5][3]),
                 "+r"(r[5][4]), "+r"(r[5][5]), "+r"(r[5][6]), "+r"(r[5][7]), "+r"(r[6][0]), "+r"(r[6][1]),
                 "+r"(r[6][2]), "+r"(r[6][3]), "+r"(r[6][4]), "+r"(r[6][5]), "+r"(r[6][6]), "+r"(r[6][7]),
                 "+r"(r[7][0]), "+r"(r[7][1]), "+r"(r[7][2]), "+r"(r[7][3]), "+r"(r[7][4]), "+r"(r[7][5]),
                 "+r"(r[7][6]), "+r"(r[7][7])
               :
               : "memory");
}
__device__ __forceinline__ void tie_regs(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// Exact three-part bf16 split of an fp32 value v >= 0: v == hi + mid + lo.
__device__ __forceinline__ void split3(float v, float& hi, float& mid, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(v));
  const float r1 = v - hi;
  mid = __bfloat162float(__float2bfloat16_rn(r1));
  lo = __bfloat162float(__float2bfloat16_rn(r1 - mid));
}
// Pad words of a row: 16-byte chunks k8 = G/8 .. KP/8-1 (6 used elements).
// A rows hold [xx_hi xx_mid xx_lo 1 1 1 0 ...], B rows [1 1 1 nc_hi nc_mid nc_lo 0 ...].
template <int KP, int G>
__device__ __forceinline__ void write_pad(uint8_t* base, int r, float a0, float a1, float a2, float b0, float b1,
                                          float b2) {
  const uint4 w0 = make_uint4(pack_bf16(a0, a1), pack_bf16(a2, b0), pack_bf16(b1, b2), 0u);
  *reinterpret_cast<uint4*>(base + core_off<KP>(r, G / 8)) = w0;
#pragma unroll
  for (int k8 = G / 8 + 1; k8 < KP / 8; ++k8) *reinterpret_cast<uint4*>(base + core_off<KP>(r, k8)) = make_uint4(0u, 0u, 0u, 0u);
}

template <int G, int KP>
__global__ void __launch_bounds__(kTcThreads, 2) encode_tc_kernel(const EncodeTcParams p) {
  extern __shared__ __align__(1024) uint8_t dyn[];
  constexpr uint32_t kBBytes = kTcCodes * KP * 2;
  constexpr uint32_t kABytes = kTcTile * KP * 2;
  uint8_t* const bsm = dyn;
  uint8_t* const asmem = dyn + kBBytes;
  uint64_t* const mbar = reinterpret_cast<uint64_t*>(dyn + kBBytes + kABytes);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(mbar + 1);
  int* const nc_max_bits = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x;
  const int bh = blockIdx.z;
  const int b = bh / p.H, h = bh % p.H;
  const int64_t tile0 = (int64_t)blockIdx.y * kTcTilesPerCta;
  const int64_t n_tiles_total = (p.n_tokens + kTcTile - 1) / kTcTile;
  const int64_t left = n_tiles_total - tile0;
  const int n_tiles = left < kTcTilesPerCta ? (int)left : kTcTilesPerCta;
  if (n_tiles <= 0) return;  // uniform across the CTA, before any allocation

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTcCodes));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    mbar_init(smem_u32(mbar), 1);
    *nc_max_bits = 0;
    fence_mbar_init();
  }

  // ---- B operand: row c = [-2c (G) | 1 1 1 nc_hi nc_mid nc_lo | 0 ...] ----
  const __nv_bfloat16* cbp = p.cb + (((int64_t)bh * p.J + j) * kTcCodes) * G;
  float ncmax = 0.f;
#pragma unroll 1
  for (int c = tid; c < kTcCodes; c += kTcThreads) {
    const uint4* src = reinterpret_cast<const uint4*>(cbp + (int64_t)c * G);
    float nc = 0.f;
#pragma unroll
    for (int k8 = 0; k8 < G / 8; ++k8) {
      const uint4 v = __ldg(src + k8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = bf16_lo(w[i]), hi = bf16_hi(w[i]);
        nc = fmaf(lo, lo, nc);
        nc = fmaf(hi, hi, nc);
        o[i] = pack_bf16(-2.f * lo, -2.f * hi);  // exact: a power-of-two scale of a bf16 value
      }
      *reinterpret_cast<uint4*>(bsm + core_off<KP>(c, k8)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    float hi, mid, lo;
    split3(nc, hi, mid, lo);
    write_pad<KP, G>(bsm, c, 1.f, 1.f, 1.f, hi, mid, lo);
    ncmax = fmaxf(ncmax, nc);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ncmax = fmaxf(ncmax, __shfl_xor_sync(0xffffffffu, ncmax, o));
  __syncthreads();  // nc_max_bits initialised
  if (lane == 0) atomicMax(nc_max_bits, __float_as_int(ncmax));  // non-negative floats order as ints
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float nc_max = __int_as_float(*nc_max_bits);
  const uint32_t a_addr = smem_u32(asmem), b_addr = smem_u32(bsm);
  const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's 32 TMEM lanes

  // ---- sub-vector loads: G/4 groups of 4 consecutive channels (W % 4 == 0) ----
  const int row = tid;
  uint2 xr[G / 4];
  int64_t n_next = tile0 * kTcTile + row;
  auto load_x = [&](int64_t n) {
#pragma unroll
    for (int q = 0; q < G / 4; ++q) {
      const int g = q * 4, t = g / p.W, w = g - t * p.W;
      xr[q] = make_uint2(0u, 0u);
      if (n < p.n_tokens)
        xr[q] = __ldg(reinterpret_cast<const uint2*>(p.x + (int64_t)(b * p.Tc + t) * p.st + n * p.sn +
                                                     (int64_t)h * p.sh + (int64_t)j * p.W + w));
    }
  };
  load_x(n_next);

  uint32_t phase = 0;
#pragma unroll 1
  for (int tile = 0; tile < n_tiles; ++tile) {
    const int64_t n = n_next;
    const bool ok = n < p.n_tokens;
    // A row: the sub-vector's bf16 words as loaded, then the norm parts
    float xx = 0.f;
#pragma unroll
    for (int k8 = 0; k8 < G / 8; ++k8) {
      const uint2 u0 = xr[2 * k8], u1 = xr[2 * k8 + 1];
      *reinterpret_cast<uint4*>(asmem + core_off<KP>(row, k8)) = make_uint4(u0.x, u0.y, u1.x, u1.y);
      const uint32_t w[4] = {u0.x, u0.y, u1.x, u1.y};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xx = fmaf(bf16_lo(w[i]), bf16_lo(w[i]), xx);
        xx = fmaf(bf16_hi(w[i]), bf16_hi(w[i]), xx);
      }
    }
    // Fast-path error bound per codeword.  Every product of two bf16 values is
    // exact in fp32, so the contraction's error is that of summing its KP
    // terms: each partial sum is at most S = sum |terms| <= 2 (||x||^2 +
    // max ||c||^2), and each of the KP - 1 additions rounds (or truncates) by at
    // most 2^-23 of it, so at most (KP - 1) 2^-22 (||x||^2 + max ||c||^2).  The
    // fp32 norm ||c||^2 (G fused multiply-adds) adds at most G 2^-24 max ||c||^2;
    // the norm ||x||^2 is the same for every codeword and cancels.
    const float err = (float)(4 * (KP - 1) + G) * 5.9604645e-8f * (xx + nc_max);
    // Keys quantize the fast distance at a power-of-two scale sk with
    // d * sk < 2^22 (d <= (|x| + |c|)^2 + 2 err <= 2 (||x||^2 + max ||c||^2) + 2 err):
    // fma(d, sk, 2^23) holds round(d * sk) in its low 23 bits, and
    // bits * 256 + column puts the column below it -- one FFMA and one
    // integer multiply-add per candidate, off the integer ALU pipe.
    int ek = (int)((__float_as_uint(2.f * (xx + nc_max) + 4.f * err) >> 23) & 0xFFu) - 127;
    ek = max(ek, -100);
    const float sk = __uint_as_float((uint32_t)(21 - ek + 127) << 23);
    const float inv_sk = __uint_as_float((uint32_t)(ek - 21 + 127) << 23);
    {
      // the row's norm carries a bias of 2 err, equal for every codeword, so
      // the fast distances stay positive and order as signed integers
      float hi, mid, lo;
      split3(xx + 2.f * err, hi, mid, lo);
      write_pad<KP, G>(asmem, row, hi, mid, lo, 1.f, 1.f, 1.f);
    }
    // generic-proxy writes of A (and, the first time, B) -> tensor core
    fence_proxy_async();
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    if (tid == 0) {
#pragma unroll
      for (int k = 0; k < KP / 16; ++k)
        umma_f16(tmem, umma_smem_desc<KP>(a_addr + k * 256), umma_smem_desc<KP>(b_addr + k * 256), k > 0 ? 1u : 0u);
      umma_commit(smem_u32(mbar));
    }
    // next tile's loads fly while the MMA runs
    n_next += kTcTile;
    if (tile + 1 < n_tiles) load_x(n_next);

    const bool done = mbar_wait_bounded(smem_u32(mbar), phase);
    if (__syncthreads_or(!done)) {
      // never expected: record it, give the MMA one more bounded wait so no
      // tensor-core write is in flight, then leave (codes of this tile unwritten)
      if (tid == 0) set_fault(p.faults, LOOPVQ_FAULT_TIMEOUT);
      mbar_wait_bounded(smem_u32(mbar), phase);
      break;
    }
    phase ^= 1u;
    tmem_fence_after();

    // Top-2 keys over the 256 codes, 64 TMEM columns at a time (the next 64
    // load while these are scanned), in 4 independent chains: chain c takes
    // the 8-column groups 32g + 8c (g = 0..7), so that its 64 columns can be
    // re-read with eight 8-column loads.  A pair (lo <= hi) merges into a
    // chain's sorted (x1 <= x2) as x2 = min(max(x1, lo), x2, hi),
    // x1 = min(x1, lo); the code is the key's low byte (an immediate).
    auto qkey = [&](uint32_t v, uint32_t code) -> int {
      const float y = __fmaf_rn(__uint_as_float(v), sk, 8388608.f);
      return (int)(__float_as_uint(y) * p.key_mul + code);
    };
    int x1[4], x2[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) { x1[c] = 0x7FFFFFFF; x2[c] = 0x7FFFFFFF; }
    uint32_t rb[2][2][32];
    tmem_ld32(t_row, rb[0][0]);
    tmem_ld32(t_row + 32u, rb[0][1]);
    tmem_wait_ld_tied(rb[0][0]);
    tie_regs(rb[0][1]);
#pragma unroll
    for (int i = 0; i < kTcCodes / 64; ++i) {
      uint32_t (&cur)[2][32] = rb[i & 1];
      uint32_t (&nxt)[2][32] = rb[(i + 1) & 1];
      if (i + 1 < kTcCodes / 64) {
        tmem_ld32(t_row + (uint32_t)(64 * i + 64), nxt[0]);
        tmem_ld32(t_row + (uint32_t)(64 * i + 96), nxt[1]);
      }
#pragma unroll
      for (int pp = 0; pp < 32; ++pp) {
        const int col = 2 * pp;
        const int k0 = qkey(cur[col >> 5][col & 31], (uint32_t)(64 * i + col));
        const int k1v = qkey(cur[(col + 1) >> 5][(col + 1) & 31], (uint32_t)(64 * i + col + 1));
        const int lo = min(k0, k1v), hi = max(k0, k1v);
        const int c = (pp >> 2) & 3;
        x2[c] = min(min(max(x1[c], lo), x2[c]), hi);
        x1[c] = min(x1[c], lo);
      }
      if (i + 1 < kTcCodes / 64) {
        tmem_wait_ld_tied(nxt[0]);
        tie_regs(nxt[1]);
      }
    }
    // the row's two smallest keys: k1 is the smallest chain head; k2 the
    // smallest of the other heads and of every chain's second
    const int k1 = min(min(x1[0], x1[1]), min(x1[2], x1[3]));
    int k2 = min(min(x2[0], x2[1]), min(x2[2], x2[3]));
#pragma unroll
    for (int c = 0; c < 4; ++c) k2 = min(k2, x1[c] != k1 ? x1[c] : 0x7FFFFFFF);
    int code = k1 & 0xFF;
    // a key is a candidate when its gap to k1 (units of 1/sk) is within twice
    // the fast path's error bound plus the keys' rounding (half a unit each)
    const float bound = 2.f * err * sk + 2.f;
    auto near = [&](int k) -> bool { return !((float)((k >> 8) - (k1 >> 8)) > bound); };
    const bool refine = ok && near(k2);
    if (__any_sync(0xffffffffu, refine)) {
      // Only codes whose fast distance is within 2 err of the minimum can be
      // the nearest.  The sorted chain values are the row's smallest keys up
      // to the first chain second within the bound (that chain's third is not
      // kept), so the candidates are the chain heads within the bound plus
      // every column of the chains whose second is within it, re-read from
      // TMEM.
      uint32_t rescan = 0;
      if (refine) {
#pragma unroll
        for (int c = 0; c < 4; ++c) rescan |= near(x2[c]) ? 1u << c : 0u;
      }
      float xe[G];
#pragma unroll
      for (int k8 = 0; k8 < G / 8; ++k8) {
        const uint4 v = *reinterpret_cast<const uint4*>(asmem + core_off<KP>(row, k8));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) { xe[k8 * 8 + 2 * i] = bf16_lo(w[i]); xe[k8 * 8 + 2 * i + 1] = bf16_hi(w[i]); }
      }
      // exact fp32 distance sum_g (x_g - c_g)^2 to codeword c
      auto exact_d = [&](int c) -> float {
        float d = 0.f;
#pragma unroll
        for (int k8 = 0; k8 < G / 8; ++k8) {
          const uint4 v = *reinterpret_cast<const uint4*>(bsm + core_off<KP>(c, k8));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // B holds -2c: c = -B/2 exactly
            const float df0 = xe[k8 * 8 + 2 * i] + 0.5f * bf16_lo(w[i]);
            const float df1 = xe[k8 * 8 + 2 * i + 1] + 0.5f * bf16_hi(w[i]);
            d = fmaf(df0, df0, d);
            d = fmaf(df1, df1, d);
          }
        }
        return d;
      };
      // the smallest exact distance, ties to the lower code
      float best = INFINITY;
      int bi = code;
      auto consider = [&](int c) {
        const float d = exact_d(c);
        if (d < best || (d == best && c < bi)) { best = d; bi = c; }
      };
      if (refine) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c)
          if (!(rescan >> c & 1u) && near(x1[c])) consider(x1[c] & 0xFF);
      }
      const float thr = (float)(k1 >> 8) * inv_sk + 2.f * err + 2.f * inv_sk;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        if (!__any_sync(0xffffffffu, rescan >> c & 1u)) continue;
        uint32_t r[8][8];
#pragma unroll
        for (int g = 0; g < 8; ++g) tmem_ld8(t_row + (uint32_t)(32 * g + 8 * c), r[g]);
        tmem_wait_ld_tied64(r);
        uint64_t cand = 0;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
#pragma unroll
          for (int q = 0; q < 8; ++q) cand |= (uint64_t)(__uint_as_float(r[g][q]) <= thr ? 1u : 0u) << (8 * g + q);
        }
        if (!(rescan >> c & 1u)) cand = 0;
        while (cand) {
          const int bit = __ffsll((long long)cand) - 1;
          cand &= cand - 1;
          consider(32 * (bit >> 3) + 8 * c + (bit & 7));
        }
      }
      if (refine) code = bi;
    }
    if (ok) p.pool[pool_byte(p.J, p.kind, p.pool_tokens, b, p.H, h, p.tok_off + n, j)] = (uint8_t)code;
    tmem_fence_before();  // TMEM reads ordered before the next tile's barrier and MMA
  }
  __syncthreads();
  tmem_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCodes));
}

template <int G>
static cudaError_t launch_encode_tc(const EncodeTcParams& p, dim3 grid, cudaStream_t s) {
  constexpr int KP = ((G + 6) + 15) / 16 * 16;
  constexpr int need = kTcCodes * KP * 2 + kTcTile * KP * 2 + 64;
  constexpr int smem = need > kTcSmemFloor ? need : kTcSmemFloor;
  auto fn = encode_tc_kernel<G, KP>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  fn<<<grid, kTcThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// Tensor-core path of loopvq_encode: bf16 sub-vectors and 256-entry bf16
// codebooks with G in {16, 32} and W a multiple of 4.  Returns false (and
// launches nothing) when the shape is not served.
bool encode_tc_try(const Geo& g, const void* cb, int kind, const void* x, int64_t n_tokens, int64_t st, int64_t sn,
                   int64_t sh, uint8_t* pool, int64_t tok_off, int64_t pool_tokens, uint32_t* faults, cudaStream_t s,
                   cudaError_t* err) {
  if (!g.cb_bf16 || g.C != kTcCodes || (g.G != 16 && g.G != 32) || (g.W & 3)) return false;
  if (((uintptr_t)x & 7) || (st & 3) || (sn & 3) || (sh & 3)) return false;
  const int64_t tiles = (n_tokens + kTcTile - 1) / kTcTile;
  const int64_t ctas_y = (tiles + kTcTilesPerCta - 1) / kTcTilesPerCta;
  if (ctas_y > 65535 || (int64_t)g.NB * g.H > 65535) return false;
  EncodeTcParams p;
  p.x = (const __nv_bfloat16*)x;
  p.st = st; p.sn = sn; p.sh = sh;
  p.n_tokens = n_tokens;
  p.cb = (const __nv_bfloat16*)cb;
  p.Tc = g.Tc; p.H = g.H; p.J = g.J; p.W = g.W; p.kind = kind;
  p.pool = pool; p.tok_off = tok_off; p.pool_tokens = pool_tokens;
  p.faults = faults;
  p.key_mul = 256u;
  // slot j fastest: the J CTAs of one token chunk run together and share its
  // sectors in L2
  dim3 grid(g.J, (unsigned)ctas_y, g.NB * g.H);
  *err = g.G == 16 ? launch_encode_tc<16>(p, grid, s) : launch_encode_tc<32>(p, grid, s);
  return true;
}

}  // namespace loopvq
