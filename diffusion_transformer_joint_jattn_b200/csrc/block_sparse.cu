// Block selection of the block-sparse joint attention.
//
// Method ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA
// Blackwell GPUs", sections "Quantized and sparse attention" and "Optimized
// single-GPU deployment"): a block-sparse attention kernel whose sparsity a
// parameter tau controls, a higher tau dropping more blocks; tau = 0 is the
// dense attention.  The page names no selection rule.  Read here as: queries
// in blocks of 256 joint tokens (one CTA of the forward kernel), keys in
// blocks of 128 (one key tile); each block is represented by the mean of its
// rotated rows; for query block I the estimated attention share of key block
// J is the softmax over J of qbar_I . kbar_J * scale; J is kept iff its share
// is at least tau / n_kb (tau times a uniform share), and the largest share
// is always kept (ties to the lower block).
//
// Two launches:
//   block_pool_kernel    column sums of every 128-token tile of Q and K
//                        (coalesced 16-byte loads, one CTA per tile);
//   block_select_kernel  one CTA per (b, h, query block): the block logits
//                        (a warp per key block), the shares, the threshold,
//                        and the kept key tiles compacted in ascending order
//                        -> kv_list / kv_count, which the forward kernel
//                        walks instead of every key tile.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "jattn.h"
#include "jattn_internal.h"

namespace jattn {

namespace {

constexpr int kPoolThreads = 128;
constexpr int kSelThreads = 128;

template <int D, bool BF16>
__global__ void __launch_bounds__(kPoolThreads) block_pool_kernel(const SparseParams p) {
  constexpr int CG = D / 8;                    // 16-byte chunks per row
  constexpr int RPP = kPoolThreads / CG;       // rows per pass
  __shared__ float part[RPP][D];
  const int blk = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const int tid = threadIdx.x, cg = tid % CG, r0 = tid / CG;
  const uint16_t* x = static_cast<const uint16_t*>(which == 0 ? p.q : p.k) + static_cast<size_t>(bh) * p.S * D;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int r = r0; r < JATTN_BLOCK; r += RPP) {
    const int t = blk * JATTN_BLOCK + r;
    if (t >= p.S) break;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * D + cg * 8));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float a, b;
      if constexpr (BF16) {
        a = __uint_as_float(w[e] << 16);
        b = __uint_as_float(w[e] & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
        a = f.x;
        b = f.y;
      }
      acc[2 * e] += a;
      acc[2 * e + 1] += b;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[r0][cg * 8 + e] = acc[e];
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RPP; ++r) s += part[r][tid];
    p.pool[((static_cast<size_t>(which) * p.BH + bh) * p.nblk + blk) * D + tid] = s;
  }
}

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kSelThreads / 32; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  return r;
}

// grid (n_qb, B*H): one query block of 256 tokens (two 128-token tiles).
// The block logits are computed a warp per key block (coalesced float4 reads
// of the key block's column sums, a shuffle reduction) into this CTA's row
// of p.logits, then read back coalesced for the max, the softmax
// denominator and the threshold.
template <int D>
__global__ void __launch_bounds__(kSelThreads) block_select_kernel(const SparseParams p) {
  constexpr int NW = kSelThreads / 32;
  constexpr int CPL = D / 32;                  // channels per lane (4 or 2)
  __shared__ __align__(16) float qbar[D];
  __shared__ float red[NW];
  __shared__ float wmx[NW];
  __shared__ int warg[NW];
  __shared__ int wcount[NW];
  const int I = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int n_qb = gridDim.x, n_kb = p.nblk;
  const int r_lo = I * 2 * JATTN_BLOCK, r_hi = min(p.S, r_lo + 2 * JATTN_BLOCK);
  const float* pq = p.pool + (static_cast<size_t>(bh) * p.nblk) * D;
  const float* pk = p.pool + (static_cast<size_t>(p.BH) + bh) * p.nblk * D;
  float* lg = p.logits + (static_cast<size_t>(bh) * n_qb + I) * n_kb;
  if (tid < D) {
    float s = pq[static_cast<size_t>(2 * I) * D + tid];
    if (2 * I + 1 < p.nblk) s += pq[static_cast<size_t>(2 * I + 1) * D + tid];
    qbar[tid] = s / static_cast<float>(r_hi - r_lo);
  }
  __syncthreads();
  // logits qbar . kbar_J * scale; the largest and its (lowest) block
  float mx = -INFINITY;
  int arg = 0x7fffffff;
  for (int J = warp; J < n_kb; J += NW) {
    const float* kr = pk + static_cast<size_t>(J) * D + lane * CPL;
    float s = 0.f;
    if constexpr (CPL == 4) {
      const float4 k4 = *reinterpret_cast<const float4*>(kr);
      const float4 q4 = *reinterpret_cast<const float4*>(qbar + lane * CPL);
      s = fmaf(q4.x, k4.x, fmaf(q4.y, k4.y, fmaf(q4.z, k4.z, q4.w * k4.w)));
    } else {
      const float2 k2 = *reinterpret_cast<const float2*>(kr);
      const float2 q2 = *reinterpret_cast<const float2*>(qbar + lane * CPL);
      s = fmaf(q2.x, k2.x, q2.y * k2.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const int n = min(p.S - J * JATTN_BLOCK, JATTN_BLOCK);
    s = s / static_cast<float>(n) * p.scale;
    if (lane == 0) lg[J] = s;
    if (s > mx) { mx = s; arg = J; }               // warp-uniform: every lane holds s
  }
  if (lane == 0) { wmx[warp] = mx; warg[warp] = arg; }
  __syncthreads();                                  // also orders the logit writes before the reads below
  mx = wmx[0];
  arg = warg[0];
#pragma unroll
  for (int w = 1; w < NW; ++w)
    if (wmx[w] > mx || (wmx[w] == mx && warg[w] < arg)) { mx = wmx[w]; arg = warg[w]; }
  // the softmax denominator
  float den = 0.f;
  for (int J = tid; J < n_kb; J += kSelThreads) den += expf(lg[J] - mx);
  den = block_reduce(den, red, false);
  // keep share >= tau / n_kb, i.e. exp(s - mx) >= den * tau / n_kb, and the
  // largest; write the kept blocks in ascending order.
  const float cut = den * p.tau / static_cast<float>(n_kb);
  int32_t* list = p.kv_list + (static_cast<size_t>(bh) * n_qb + I) * n_kb;
  int base = 0;
  for (int J0 = 0; J0 < n_kb; J0 += kSelThreads) {
    const int J = J0 + tid;
    bool keep = false;
    if (J < n_kb) keep = J == arg || expf(lg[J] - mx) >= cut;
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) wcount[warp] = __popc(bal);
    __syncthreads();
    int off = base;
    for (int w = 0; w < warp; ++w) off += wcount[w];
    if (keep) list[off + __popc(bal & ((1u << lane) - 1u))] = J;
    int tot = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) tot += wcount[w];
    base += tot;
    __syncthreads();
  }
  if (tid == 0) p.kv_count[static_cast<size_t>(bh) * n_qb + I] = base;
}

}  // namespace

cudaError_t launch_block_select(const SparseParams& p, bool in_bf16, cudaStream_t st) {
  dim3 gp(p.nblk, p.BH, 2);
  if (p.d == 128) {
    if (in_bf16) block_pool_kernel<128, true><<<gp, kPoolThreads, 0, st>>>(p);
    else block_pool_kernel<128, false><<<gp, kPoolThreads, 0, st>>>(p);
  } else {
    if (in_bf16) block_pool_kernel<64, true><<<gp, kPoolThreads, 0, st>>>(p);
    else block_pool_kernel<64, false><<<gp, kPoolThreads, 0, st>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 gs(p.n_qb, p.BH);
  if (p.d == 128) block_select_kernel<128><<<gs, kSelThreads, 0, st>>>(p);
  else block_select_kernel<64><<<gs, kSelThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace jattn
