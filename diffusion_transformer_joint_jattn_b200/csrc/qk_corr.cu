// Correction operands of the high-precision 16-bit path.
//
// The 16-bit path rounds the rotated queries and keys to fp16 before the
// Q.K^T product.  The rounding error of one channel pair's contribution to a
// logit is proportional to |q_pair| |k_pair|, so it is concentrated in the
// pairs whose magnitude stands out (activation outliers: a few channels of a
// head scaled far above the rest).  For each (batch, head) this file
//   1. picks the NSEL pairs with the largest max_i |q_i,pair|^2 * max_j |k_j,pair|^2
//      (the prologue left the per-block maxima in pair_stat; ties go to the
//      lower pair index), and
//   2. writes, for every token, the fp16 high and low parts of those pairs'
//      rotated values, x = hi + lo with hi = fp16(x) (the value the prologue
//      stored) and lo = fp16(x - hi), as one 16-channel row per token:
//        Q row [hi(c_0..c_7) | lo(c_0..c_7)],  K row [lo(c_0..c_7) | hi(c_0..c_7)],
//      so that Qc . Kc^T = sum over the selected channels of
//      hi_q lo_k + lo_q hi_k: the terms the fp16 product left out, up to
//      lo_q lo_k (relative size 2^-22).
// The forward kernel adds Qc . Kc^T into each logit tile with one more
// 16-deep MMA.  Values are recomputed from the inputs with the prologue's own
// arithmetic (rope_math.cuh), so hi equals the stored fp16 value bit for bit.
//
// The page ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA
// Blackwell GPUs", section "Quantized and sparse attention") runs BF16
// attention as the accuracy reference; this correction is how this library
// keeps its 16-bit tensor-core operands within the BF16 path's error bars.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "jattn.h"
#include "jattn_internal.h"
#include "rope_math.cuh"

namespace jattn {

namespace {

constexpr int kSelThreads = 256;

// One CTA per (b, h): reduce the per-block pair maxima of Q and K, then take
// the NSEL largest products (a warp argmax, NSEL times).  Output: the pair
// indices in ascending order.
template <int D>
__global__ void __launch_bounds__(kSelThreads) qk_select_kernel(const CorrParams p) {
  constexpr int NPAIR = D / 2;
  constexpr int PARTS = kSelThreads / NPAIR;          // threads per pair (4 for d = 128, 8 for d = 64)
  __shared__ float pa[PARTS][NPAIR], pc[PARTS][NPAIR];
  __shared__ float prod[NPAIR];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  const size_t plane = static_cast<size_t>(p.BH) * p.nblk * NPAIR;
  const float* sq = p.pair_stat + static_cast<size_t>(bh) * p.nblk * NPAIR;
  const float* sk = sq + plane;
  {
    // PARTS threads per pair, strided over the blocks (consecutive threads
    // read consecutive pairs of one block).
    const int pair = tid % NPAIR, part = tid / NPAIR;
    float a = 0.f, c = 0.f;
    for (int blk = part; blk < p.nblk; blk += PARTS) {
      a = fmaxf(a, sq[static_cast<size_t>(blk) * NPAIR + pair]);
      c = fmaxf(c, sk[static_cast<size_t>(blk) * NPAIR + pair]);
    }
    pa[part][pair] = a;
    pc[part][pair] = c;
  }
  __syncthreads();
  if (tid < NPAIR) {
    float a = 0.f, c = 0.f;
#pragma unroll
    for (int k = 0; k < PARTS; ++k) {
      a = fmaxf(a, pa[k][tid]);
      c = fmaxf(c, pc[k][tid]);
    }
    prod[tid] = a * c;
  }
  __syncthreads();
  if (tid < 32) {
    int chosen[kCorrPairs];
#pragma unroll
    for (int k = 0; k < kCorrPairs; ++k) {
      float best = -1.f;
      int arg = NPAIR;
      for (int q = tid; q < NPAIR; q += 32) {
        bool taken = false;
#pragma unroll
        for (int m = 0; m < k; ++m) taken |= chosen[m] == q;
        const float v = taken ? -1.f : prod[q];
        if (v > best || (v == best && q < arg)) { best = v; arg = q; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
        if (ob > best || (ob == best && oa < arg)) { best = ob; arg = oa; }
      }
      chosen[k] = arg;
    }
    if (tid == 0) {
#pragma unroll
      for (int a = 1; a < kCorrPairs; ++a)
#pragma unroll
        for (int c = a; c > 0; --c)
          if (chosen[c - 1] > chosen[c]) { const int t = chosen[c]; chosen[c] = chosen[c - 1]; chosen[c - 1] = t; }
#pragma unroll
      for (int k = 0; k < kCorrPairs; ++k) p.sel[static_cast<size_t>(bh) * kCorrPairs + k] = chosen[k];
    }
  }
}

__device__ __forceinline__ uint32_t pack_h2(__half a, __half b) {
  return static_cast<uint32_t>(__half_as_ushort(a)) | (static_cast<uint32_t>(__half_as_ushort(b)) << 16);
}

// grid (nblk, B*H), one thread per token of the block.
template <int D, bool NORM>
__global__ void __launch_bounds__(JATTN_BLOCK) qk_correct_kernel(const CorrParams p) {
  const int blk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const int t = blk * JATTN_BLOCK + threadIdx.x;
  if (t >= p.S) return;
  int stream = 0, local = t;
  if (t >= p.S_part[0]) { stream = 1; local = t - p.S_part[0]; }
  if (t >= p.S_part[0] + p.S_part[1]) { stream = 2; local = t - p.S_part[0] - p.S_part[1]; }
  const __nv_bfloat16* row = p.src[stream] + (static_cast<size_t>(b) * p.S_part[stream] + local) * 3 * p.H * D;
  int pairs[kCorrPairs];
#pragma unroll
  for (int k = 0; k < kCorrPairs; ++k) pairs[k] = p.sel[static_cast<size_t>(bh) * kCorrPairs + k];
  float cs[kCorrPairs], sn[kCorrPairs];
#pragma unroll
  for (int k = 0; k < kCorrPairs; ++k)
    angle_cos_sin(p.pos[3 * t + p.rope.axis[pairs[k]]], p.rope.omega[pairs[k]], cs[k], sn[k]);
  const size_t BHS = static_cast<size_t>(p.BH) * p.S;
  // All eight channel-pair words (Q and K) are requested before any is used.
  uint32_t words[2][kCorrPairs];
#pragma unroll
  for (int which = 0; which < 2; ++which)
#pragma unroll
    for (int k = 0; k < kCorrPairs; ++k)
      words[which][k] = __ldg(reinterpret_cast<const uint32_t*>(row + (which * p.H + h) * D) + pairs[k]);
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const float inv2e = 1.0f / p.scales[(static_cast<size_t>(which) * p.BH + bh) * p.nblk + blk];
    float r = 1.f;
    if constexpr (NORM) r = p.norm_r[which * BHS + static_cast<size_t>(bh) * p.S + t];
    __half hi[2 * kCorrPairs], lo[2 * kCorrPairs];
#pragma unroll
    for (int k = 0; k < kCorrPairs; ++k) {
      const uint32_t u = words[which][k];                            // channels 2p, 2p + 1
      float a = bf16_to_f32(static_cast<uint16_t>(u & 0xFFFFu));
      float c = bf16_to_f32(static_cast<uint16_t>(u >> 16));
      if constexpr (NORM) {
        const float* w = p.norm_w + (stream * 2 + which) * D + 2 * pairs[k];
        a = norm_scale(a, r, w[0]);
        c = norm_scale(c, r, w[1]);
      }
      float x0, x1;
      rotate_pair(a, c, cs[k], sn[k], x0, x1);
      x0 = __fmul_rn(x0, inv2e);
      x1 = __fmul_rn(x1, inv2e);
      hi[2 * k] = __float2half_rn(x0);
      hi[2 * k + 1] = __float2half_rn(x1);
      lo[2 * k] = __float2half_rn(x0 - __half2float(hi[2 * k]));          // exact difference
      lo[2 * k + 1] = __float2half_rn(x1 - __half2float(hi[2 * k + 1]));
    }
    const uint4 vh = make_uint4(pack_h2(hi[0], hi[1]), pack_h2(hi[2], hi[3]), pack_h2(hi[4], hi[5]),
                                pack_h2(hi[6], hi[7]));
    const uint4 vl = make_uint4(pack_h2(lo[0], lo[1]), pack_h2(lo[2], lo[3]), pack_h2(lo[4], lo[5]),
                                pack_h2(lo[6], lo[7]));
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(which == 0 ? p.qc : p.kc) +
                                          (static_cast<size_t>(bh) * p.S + t) * kCorrCols);
    dst[0] = which == 0 ? vh : vl;
    dst[1] = which == 0 ? vl : vh;
  }
}

}  // namespace

cudaError_t launch_qk_correction(const CorrParams& p, cudaStream_t st) {
  if (p.d == 128) {
    qk_select_kernel<128><<<p.BH, kSelThreads, 0, st>>>(p);
  } else {
    qk_select_kernel<64><<<p.BH, kSelThreads, 0, st>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid(p.nblk, p.BH);
  if (p.d == 128) {
    if (p.norm_w != nullptr) qk_correct_kernel<128, true><<<grid, JATTN_BLOCK, 0, st>>>(p);
    else qk_correct_kernel<128, false><<<grid, JATTN_BLOCK, 0, st>>>(p);
  } else {
    if (p.norm_w != nullptr) qk_correct_kernel<64, true><<<grid, JATTN_BLOCK, 0, st>>>(p);
    else qk_correct_kernel<64, false><<<grid, JATTN_BLOCK, 0, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace jattn
