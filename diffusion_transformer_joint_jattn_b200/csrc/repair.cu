// Token selection for the FP8 attention with repair ("Speed Up Image
// Generation with FLUX 3 Image Klein on NVIDIA Blackwell GPUs", section
// "Quantized and sparse attention": a repair budget rho selects the fraction
// of tokens with the highest quantisation error for a residual correction).
//
// Per (batch, head) the n tokens with the largest score |k|^2 + |v|^2 (the
// e4m3 error bound of a token's key and value rows grows with their
// magnitude) are selected, ties going to the lower token index, and listed
// in index order; their bits are set in the key mask that the FP8 pass uses
// to leave them out.
//
// One CTA per (b, h).  Scores are non-negative floats, so their bit patterns
// order like unsigned integers: four 8-bit radix passes over the scores
// (read from L2) find the bit pattern T of the n-th largest score and how many
// of the scores equal to T are still needed; a block-wide scan then writes
// the selected indices in index order.
#include <cstdint>
#include <cuda_runtime.h>

#include "jattn.h"
#include "jattn_internal.h"

namespace jattn {

namespace {

constexpr int kSelThreads = 1024;

// Exclusive prefix sum over the block; returns this thread's prefix, and the
// total through `total`.
__device__ uint32_t block_exclusive_scan(uint32_t x, uint32_t* warp_sums, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kSelThreads / 32 ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;                             // inclusive over warps
  }
  __syncthreads();
  total = warp_sums[kSelThreads / 32 - 1];
  const uint32_t before = warp == 0 ? 0u : warp_sums[warp - 1];
  __syncthreads();                                   // warp_sums is reused by the next scan
  return before + incl - x;
}

// score: [2][B*H][S], the |k|^2 plane then the |v|^2 plane; the K plane is
// overwritten with the sums.
__global__ void __launch_bounds__(kSelThreads) repair_select_kernel(float* score, int S, int n, int n_kv,
                                                                    int32_t* __restrict__ idx,
                                                                    uint32_t* __restrict__ kmask) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_prefix, s_rank;
  const int tid = threadIdx.x;
  const size_t bh = blockIdx.x;
  float* sk = score + bh * S;
  const float* sv = score + static_cast<size_t>(gridDim.x) * S + bh * S;
  for (int i = tid; i < S; i += kSelThreads) sk[i] = sk[i] + sv[i];
  uint32_t* mask = kmask + bh * static_cast<size_t>(n_kv) * 4;
  for (int w = tid; w < n_kv * 4; w += kSelThreads) mask[w] = 0u;
  __syncthreads();
  const uint32_t* sc = reinterpret_cast<const uint32_t*>(sk);

  // Radix select: after the pass for bits [shift, shift+8), `prefix` holds the
  // top bits of T and `rank` the position (1-based, from the top) of T among
  // the scores sharing those bits.
  uint32_t prefix = 0u, pmask = 0u, rank = static_cast<uint32_t>(n);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < S; i += kSelThreads) {
      const uint32_t u = sc[i];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0u;
      int bin = 255;
      for (; bin > 0; --bin) {
        if (cum + hist[bin] >= rank) break;
        cum += hist[bin];
      }
      s_prefix = prefix | (static_cast<uint32_t>(bin) << shift);
      s_rank = rank - cum;
    }
    __syncthreads();
    prefix = s_prefix;
    rank = s_rank;
    pmask |= 255u << shift;
  }
  const uint32_t T = prefix;          // the n-th largest score's bits
  const uint32_t need_eq = rank;      // scores equal to T to take (lowest indices first)

  // Ordered compaction over contiguous chunks.
  const int chunk = (S + kSelThreads - 1) / kSelThreads;
  const int lo = min(S, tid * chunk), hi = min(S, lo + chunk);
  uint32_t gt = 0u, eq = 0u;
  for (int i = lo; i < hi; ++i) {
    const uint32_t u = sc[i];
    gt += u > T;
    eq += u == T;
  }
  uint32_t total;
  const uint32_t eq_before = block_exclusive_scan(eq, warp_sums, total);
  const uint32_t take_eq = eq_before >= need_eq ? 0u : min(eq, need_eq - eq_before);
  uint32_t pos = block_exclusive_scan(gt + take_eq, warp_sums, total);
  uint32_t eq_seen = 0u;
  for (int i = lo; i < hi; ++i) {
    const uint32_t u = sc[i];
    bool sel = u > T;
    if (u == T) {
      sel = eq_seen < take_eq;
      ++eq_seen;
    }
    if (sel && pos < static_cast<uint32_t>(n)) {
      idx[bh * n + pos] = i;
      atomicOr(&mask[i >> 5], 1u << (i & 31));
      ++pos;
    }
  }
}

}  // namespace

cudaError_t launch_repair_select(float* score, int BH, int S, int n, int n_kv, int32_t* idx,
                                 uint32_t* kmask, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  repair_select_kernel<<<BH, kSelThreads, 0, st>>>(score, S, n, n_kv, idx, kmask);
  return cudaGetLastError();
}

}  // namespace jattn
