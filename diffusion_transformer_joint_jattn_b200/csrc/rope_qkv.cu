// Prologue kernels: joint-sequence assembly + (optional query/key RMSNorm) +
// 2D axial RoPE on Q/K, with the output either in a 16-bit type or quantised
// to e4m3 with one fp32 scale per (batch, head, 128-token block); and the
// standalone block quantiser.
//
// Method ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA
// Blackwell GPUs"): the text, target-image and reference-image streams are
// joined for joint attention (section "FLUX 3 inference with TensorRT LLM
// VisualGen"); rotary embeddings act on the query and key projections, which
// the same fused projection also normalises (section "GEMM kernel
// optimization"); FP8 Q/K/V feed the quantised attention (section "Quantized
// and sparse attention").  The normalisation is taken as RMSNorm over the d
// channels of one (token, head), w * x / sqrt(mean(x^2) + eps), with one
// weight vector per stream and per Q/K, applied before the rotation.
//
// Design: HBM-bound streaming.  One CTA owns one 128-token block of one batch
// entry and walks all 3*H (Q/K/V, head) tiles of it, so each (token, pair)
// cos/sin is computed once per CTA and lives in registers; loads and stores
// are 16-byte vectors, coalesced along d; the next tile's loads are issued
// before the current tile is processed, and the one after it is prefetched
// into L2.  For e4m3 output the tile's amax is
// reduced across the CTA before its codes are written, so every input byte is
// read exactly once.  The RMSNorm's sum of squares is a shuffle reduction over
// the D/8 consecutive lanes that hold one row; its weights are staged in
// shared memory once per CTA.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "jattn.h"
#include "jattn_internal.h"
#include "rope_math.cuh"

namespace jattn {

namespace {

constexpr int kTok = JATTN_BLOCK;   // tokens per CTA (= FP8 scale block)
constexpr int kTokPerThread = 4;

enum OutKind { kOutF16 = 0, kOutBF16 = 1, kOutE4M3 = 2 };

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Two fp32 -> two e4m3 (RNE, saturating to +-448); `a` lands in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// OUT: output kind.  D: head dimension.  NORM: RMSNorm Q and K first.
// REPAIR (e4m3 output only): also write fp16 Q and the per-token repair score
// |k|^2 + |v|^2 of the values that are quantised.
// HP (fp16 output only), the high-precision 16-bit path: every (Q|K|V, head)
// tile is stored scaled by a power of two 2^-e chosen from the tile's amax
// so that nothing saturates (e = 0 unless the tile reaches past 65504; the
// scale 2^e goes to p.scales, [3][B][H][nblk]); for Q and K the maximum
// squared norm of every channel pair over the block's tokens goes to
// p.pair_stat ([2][B*H][nblk][D/2]), and with NORM each row's RMSNorm factor
// to p.norm_r ([2][B*H][S]), for the correction operands built afterwards.
template <int D, int OUT, bool NORM, bool REPAIR, bool HP>
__global__ void __launch_bounds__(D / 8 * kTok / kTokPerThread)
rope_qkv_kernel(const RopeParams p) {
  constexpr int CG = D / 8;                           // 16-byte chunks per row
  constexpr int NT = CG * kTok / kTokPerThread;       // threads
  constexpr int ROWS_PER_PASS = kTok / kTokPerThread; // tokens covered by one pass
  constexpr int NWARP = NT / 32;
  constexpr int NPAIR = D / 2;
  static_assert(CG <= 32 && 32 % CG == 0, "a row's lanes must sit inside one warp");
  static_assert(!HP || OUT == kOutF16, "the high-precision path stores fp16");
  __shared__ float red[2][NWARP];
  __shared__ __align__(16) float wsm[NORM ? 6 * D : 4];   // [stream][q/k][D]
  __shared__ __align__(16) float pst[HP ? 2 : 1][HP ? NWARP : 1][HP ? NPAIR : 4];   // pair statistics per warp

  const int tid = threadIdx.x;
  const int cg = tid % CG;
  const int trow = tid / CG;
  const int warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x;
  const int b = blockIdx.y;
  const int H = p.H, S = p.S;
  if constexpr (NORM) {
    for (int i = tid; i < 6 * D; i += NT) wsm[i] = p.norm_w[i];
    __syncthreads();
  }

  // Per-token source row base (element offset of [b, local, 0, 0, 0] in its
  // stream) and validity.
  const __nv_bfloat16* src[kTokPerThread];
  int tok[kTokPerThread];
  int stream[kTokPerThread];
  bool valid[kTokPerThread];
  float cs[kTokPerThread][4], sn[kTokPerThread][4];
#pragma unroll
  for (int i = 0; i < kTokPerThread; ++i) {
    const int t = blk * kTok + trow + i * ROWS_PER_PASS;
    tok[i] = t;
    valid[i] = t < S;
    const __nv_bfloat16* base = p.src[0];
    int len = p.S_part[0], local = t;
    stream[i] = 0;
    if (t >= p.S_part[0]) { base = p.src[1]; len = p.S_part[1]; local = t - p.S_part[0]; stream[i] = 1; }
    if (t >= p.S_part[0] + p.S_part[1]) {
      base = p.src[2]; len = p.S_part[2]; local = t - p.S_part[0] - p.S_part[1]; stream[i] = 2;
    }
    src[i] = valid[i] ? base + (static_cast<size_t>(b) * len + local) * 3 * H * D + cg * 8 : nullptr;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      cs[i][j] = 1.f;
      sn[i][j] = 0.f;
      if (valid[i]) {
        const int pair = cg * 4 + j;
        angle_cos_sin(p.pos[3 * t + p.rope.axis[pair]], p.rope.omega[pair], cs[i][j], sn[i][j]);
      }
    }
  }

  const int items = 3 * H;
  uint4 nxt[kTokPerThread];
  auto load_item = [&](int item, uint4 (&buf)[kTokPerThread]) {
    const int which = item / H, h = item % H;
    const size_t off = static_cast<size_t>(which * H + h) * D;
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i)
      buf[i] = valid[i] ? __ldg(reinterpret_cast<const uint4*>(src[i] + off)) : make_uint4(0, 0, 0, 0);
  };
  // The tile after the one held in registers is asked into L2 ahead of its
  // load: one 512-thread CTA per SM keeps too few bytes in flight with the
  // register prefetch alone.  One lane per 128-byte line issues it.
  auto prefetch_item_l2 = [&](int item) {
    const int which = item / H, h = item % H;
    const size_t off = static_cast<size_t>(which * H + h) * D;
    if ((cg & 7) == 0) {
#pragma unroll
      for (int i = 0; i < kTokPerThread; ++i)
        if (valid[i]) asm volatile("prefetch.global.L2 [%0];" ::"l"(src[i] + off));
    }
  };
  load_item(0, nxt);
  if (items > 1) prefetch_item_l2(1);
  bool range_hit = false;

  for (int item = 0; item < items; ++item) {
    uint4 cur[kTokPerThread];
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) cur[i] = nxt[i];
    if (item + 1 < items) load_item(item + 1, nxt);
    if (item + 2 < items) prefetch_item_l2(item + 2);
    const int which = item / H, h = item % H;
    const size_t row0 = (static_cast<size_t>(b) * H + h) * S;

    float x[kTokPerThread][8];
#pragma unroll
    for (int i = 0; i < kTokPerThread; ++i) {
      bf16x8_to_f32(cur[i], x[i]);
      if (NORM && which < 2) {
        // RMSNorm over the row's D channels: this thread holds 8 of them,
        // the row's other chunks sit in the CG consecutive lanes around it.
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = __fmaf_rn(x[i][e], x[i][e], ss);
#pragma unroll
        for (int o = CG / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float r = norm_factor(ss, D, p.eps);
        const float4* wv = reinterpret_cast<const float4*>(wsm + (stream[i] * 2 + which) * D + cg * 8);
        const float4 w0 = wv[0], w1 = wv[1];
        const float wr[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) x[i][e] = norm_scale(x[i][e], r, wr[e]);
        if constexpr (HP) {
          if (cg == 0 && valid[i]) p.norm_r[static_cast<size_t>(which) * p.B * H * S + row0 + tok[i]] = r;
        }
      }
      if (which < 2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) rotate_pair(x[i][2 * j], x[i][2 * j + 1], cs[i][j], sn[i][j], x[i][2 * j],
                                                x[i][2 * j + 1]);
      }
    }

    if constexpr (REPAIR) {
      if (which == 0) {
        uint16_t* q16 = static_cast<uint16_t*>(p.q16);
#pragma unroll
        for (int i = 0; i < kTokPerThread; ++i) {
          if (!valid[i]) continue;
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            y[e] = x[i][e];
            if (fabsf(y[e]) > 65504.f) {
              range_hit = true;
              y[e] = copysignf(65504.f, y[e]);
            }
          }
          *reinterpret_cast<uint4*>(q16 + (row0 + tok[i]) * D + cg * 8) =
              make_uint4(pack_f16(y[0], y[1]), pack_f16(y[2], y[3]), pack_f16(y[4], y[5]), pack_f16(y[6], y[7]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < kTokPerThread; ++i) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) ss = fmaf(x[i][e], x[i][e], ss);
#pragma unroll
          for (int o = CG / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (cg == 0 && valid[i]) {
            // K and V terms go to separate planes (the selection adds them):
            // no pass waits on a read of what an earlier one wrote.
            const size_t plane = which == 2 ? static_cast<size_t>(p.B) * H * S : 0;
            p.score[plane + row0 + tok[i]] = ss;
          }
        }
      }
    }

    if constexpr (OUT == kOutE4M3) {
      float am = 0.f;
#pragma unroll
      for (int i = 0; i < kTokPerThread; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(x[i][e]));
      am = warp_max(am);
      float* slot = red[item & 1];
      if ((tid & 31) == 0) slot[tid >> 5] = am;
      __syncthreads();
      am = 0.f;
#pragma unroll
      for (int w = 0; w < NWARP; ++w) am = fmaxf(am, slot[w]);
      const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
      const float inv = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
      uint8_t* dst = static_cast<uint8_t*>(which == 0 ? p.dst[0] : (which == 1 ? p.dst[1] : p.dst[2]));
#pragma unroll
      for (int i = 0; i < kTokPerThread; ++i) {
        if (!valid[i]) continue;
        uint2 o;
        o.x = pack_e4m3x2(__fmul_rn(x[i][0], inv), __fmul_rn(x[i][1], inv)) |
              (pack_e4m3x2(__fmul_rn(x[i][2], inv), __fmul_rn(x[i][3], inv)) << 16);
        o.y = pack_e4m3x2(__fmul_rn(x[i][4], inv), __fmul_rn(x[i][5], inv)) |
              (pack_e4m3x2(__fmul_rn(x[i][6], inv), __fmul_rn(x[i][7], inv)) << 16);
        *reinterpret_cast<uint2*>(dst + (row0 + tok[i]) * D + cg * 8) = o;
      }
      if (tid == 0)
        p.scales[((static_cast<size_t>(which) * p.B + b) * H + h) * p.nblk + blk] = scale;
    } else {
      float inv2e = 1.0f;
      if constexpr (HP) {
        // The tile's amax -> power-of-two range scale; for Q and K the
        // per-pair maximum squared norm over the block's tokens.
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < kTokPerThread; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(x[i][e]));
        am = warp_max(am);
        if (lane == 0) red[item & 1][warp] = am;
        if (which < 2) {
          float pn[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            pn[j] = 0.f;
#pragma unroll
            for (int i = 0; i < kTokPerThread; ++i)
              pn[j] = fmaxf(pn[j], __fmaf_rn(x[i][2 * j], x[i][2 * j], __fmul_rn(x[i][2 * j + 1], x[i][2 * j + 1])));
#pragma unroll
            for (int o = CG; o < 32; o <<= 1) pn[j] = fmaxf(pn[j], __shfl_xor_sync(0xffffffffu, pn[j], o));
          }
          if (lane < CG)
            *reinterpret_cast<float4*>(&pst[item & 1][warp][cg * 4]) = make_float4(pn[0], pn[1], pn[2], pn[3]);
        }
        __syncthreads();
        am = 0.f;
#pragma unroll
        for (int w = 0; w < NWARP; ++w) am = fmaxf(am, red[item & 1][w]);
        const int e2 = f16_range_exponent(am);
        inv2e = ldexpf(1.0f, -e2);
        if (tid == 0) p.scales[((static_cast<size_t>(which) * p.B + b) * H + h) * p.nblk + blk] = ldexpf(1.0f, e2);
        if (which < 2 && tid < NPAIR) {
          float m = 0.f;
#pragma unroll
          for (int w = 0; w < NWARP; ++w) m = fmaxf(m, pst[item & 1][w][tid]);
          p.pair_stat[((static_cast<size_t>(which) * p.B * H + b * H + h) * p.nblk + blk) * NPAIR + tid] = m;
        }
      }
      uint16_t* dst = static_cast<uint16_t*>(which == 0 ? p.dst[0] : (which == 1 ? p.dst[1] : p.dst[2]));
#pragma unroll
      for (int i = 0; i < kTokPerThread; ++i) {
        if (!valid[i]) continue;
        uint4 o;
        if constexpr (OUT == kOutF16) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if constexpr (HP) {
              x[i][e] = __fmul_rn(x[i][e], inv2e);            // exact: a power of two
            } else {
              const float a = fabsf(x[i][e]);
              if (a > 65504.f) {
                range_hit = true;
                x[i][e] = copysignf(65504.f, x[i][e]);
              }
            }
          }
          o.x = pack_f16(x[i][0], x[i][1]); o.y = pack_f16(x[i][2], x[i][3]);
          o.z = pack_f16(x[i][4], x[i][5]); o.w = pack_f16(x[i][6], x[i][7]);
        } else {
          o.x = pack_bf16(x[i][0], x[i][1]); o.y = pack_bf16(x[i][2], x[i][3]);
          o.z = pack_bf16(x[i][4], x[i][5]); o.w = pack_bf16(x[i][6], x[i][7]);
        }
        *reinterpret_cast<uint4*>(dst + (row0 + tok[i]) * D + cg * 8) = o;
      }
    }
  }
  if (range_hit) atomicOr(p.status, JATTN_DEV_RANGE);
}

// Standalone per-block quantiser of a laid-out [B, H, S, D] 16-bit tensor.
template <int D, bool IN_BF16>
__global__ void __launch_bounds__(D / 8 * kTok / kTokPerThread)
quant_fp8_kernel(const QuantParams p) {
  constexpr int CG = D / 8;
  constexpr int NT = CG * kTok / kTokPerThread;
  constexpr int ROWS_PER_PASS = kTok / kTokPerThread;
  constexpr int NWARP = NT / 32;
  __shared__ float red[NWARP];
  const int tid = threadIdx.x;
  const int cg = tid % CG, trow = tid / CG;
  const int blk = blockIdx.x;
  const size_t bh = blockIdx.y;
  const uint16_t* x = static_cast<const uint16_t*>(p.x) + bh * p.S * D;

  float v[kTokPerThread][8];
  bool valid[kTokPerThread];
  int tok[kTokPerThread];
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < kTokPerThread; ++i) {
    tok[i] = blk * kTok + trow + i * ROWS_PER_PASS;
    valid[i] = tok[i] < p.S;
    uint4 u = valid[i] ? __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(tok[i]) * D + cg * 8))
                       : make_uint4(0, 0, 0, 0);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (IN_BF16) {
        v[i][2 * e] = __uint_as_float(w[e] << 16);
        v[i][2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      } else {
        __half2 h2 = *reinterpret_cast<const __half2*>(&w[e]);
        float2 f = __half22float2(h2);
        v[i][2 * e] = f.x;
        v[i][2 * e + 1] = f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(v[i][e]));
  }
  am = warp_max(am);
  if ((tid & 31) == 0) red[tid >> 5] = am;
  __syncthreads();
  am = 0.f;
#pragma unroll
  for (int w = 0; w < NWARP; ++w) am = fmaxf(am, red[w]);
  const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
  const float inv = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
  uint8_t* y = static_cast<uint8_t*>(p.x8) + bh * p.S * D;
#pragma unroll
  for (int i = 0; i < kTokPerThread; ++i) {
    if (!valid[i]) continue;
    uint2 o;
    o.x = pack_e4m3x2(__fmul_rn(v[i][0], inv), __fmul_rn(v[i][1], inv)) |
          (pack_e4m3x2(__fmul_rn(v[i][2], inv), __fmul_rn(v[i][3], inv)) << 16);
    o.y = pack_e4m3x2(__fmul_rn(v[i][4], inv), __fmul_rn(v[i][5], inv)) |
          (pack_e4m3x2(__fmul_rn(v[i][6], inv), __fmul_rn(v[i][7], inv)) << 16);
    *reinterpret_cast<uint2*>(y + static_cast<size_t>(tok[i]) * D + cg * 8) = o;
  }
  if (tid == 0) p.scales[bh * p.nblk + blk] = scale;
}

// Exact keys and values of the repaired tokens: one warp per (token, b, h);
// the key row is (normalised and) rotated with the prologue's arithmetic and
// both rows are stored as fp16.
template <int D>
__global__ void __launch_bounds__(256) repair_gather_kernel(const GatherParams p) {
  constexpr int CPL = D / 32;                        // channels per lane (4 or 2)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  const int bh = blockIdx.y;
  if (r >= p.n) return;
  const int b = bh / p.H, h = bh % p.H;
  const int t = p.idx[static_cast<size_t>(bh) * p.n + r];
  if (t < 0 || t >= p.S) {                           // not produced by the selection: report, write nothing
    if (lane == 0) atomicOr(p.status, JATTN_DEV_CHECK);
    return;
  }
  int stream = 0, local = t;
  if (t >= p.S_part[0]) { stream = 1; local = t - p.S_part[0]; }
  if (t >= p.S_part[0] + p.S_part[1]) { stream = 2; local = t - p.S_part[0] - p.S_part[1]; }
  const __nv_bfloat16* row = p.src[stream] + (static_cast<size_t>(b) * p.S_part[stream] + local) * 3 * p.H * D;
  const int c0 = lane * CPL;
  float k[CPL], v[CPL];
  {
    const uint16_t* kr = reinterpret_cast<const uint16_t*>(row + (1 * p.H + h) * D + c0);
    const uint16_t* vr = reinterpret_cast<const uint16_t*>(row + (2 * p.H + h) * D + c0);
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      k[e] = __uint_as_float(static_cast<uint32_t>(kr[e]) << 16);
      v[e] = __uint_as_float(static_cast<uint32_t>(vr[e]) << 16);
    }
  }
  if (p.norm_w != nullptr) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) ss = __fmaf_rn(k[e], k[e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rr = norm_factor(ss, D, p.eps);
    const float* w = p.norm_w + (stream * 2 + 1) * D + c0;
#pragma unroll
    for (int e = 0; e < CPL; ++e) k[e] = norm_scale(k[e], rr, w[e]);
  }
#pragma unroll
  for (int j = 0; j < CPL / 2; ++j) {
    const int pair = c0 / 2 + j;
    float cs, sn;
    angle_cos_sin(p.pos[3 * t + p.rope.axis[pair]], p.rope.omega[pair], cs, sn);
    rotate_pair(k[2 * j], k[2 * j + 1], cs, sn, k[2 * j], k[2 * j + 1]);
  }
  bool range_hit = false;
  uint32_t kw[CPL / 2], vw[CPL / 2];
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    if (fabsf(k[e]) > 65504.f) { range_hit = true; k[e] = copysignf(65504.f, k[e]); }
    if (fabsf(v[e]) > 65504.f) { range_hit = true; v[e] = copysignf(65504.f, v[e]); }
  }
#pragma unroll
  for (int j = 0; j < CPL / 2; ++j) {
    kw[j] = pack_f16(k[2 * j], k[2 * j + 1]);
    vw[j] = pack_f16(v[2 * j], v[2 * j + 1]);
  }
  // The FP8 pass sees this token's key and value as zero codes: its logit is
  // exactly 0 and it adds nothing to O (the pass removes its probability
  // from the row sum, see the key mask in the forward kernel).
  {
    const size_t off8 = (static_cast<size_t>(bh) * p.S + t) * D + c0;
    if constexpr (CPL == 4) {
      *reinterpret_cast<uint32_t*>(p.k8 + off8) = 0u;
      *reinterpret_cast<uint32_t*>(p.v8 + off8) = 0u;
    } else {
      *reinterpret_cast<uint16_t*>(p.k8 + off8) = 0u;
      *reinterpret_cast<uint16_t*>(p.v8 + off8) = 0u;
    }
  }
  const size_t off = (static_cast<size_t>(bh) * p.n + r) * D + c0;
  uint16_t* ko = static_cast<uint16_t*>(p.k_out) + off;
  uint16_t* vo = static_cast<uint16_t*>(p.v_out) + off;
  if constexpr (CPL == 4) {
    *reinterpret_cast<uint2*>(ko) = make_uint2(kw[0], kw[1]);
    *reinterpret_cast<uint2*>(vo) = make_uint2(vw[0], vw[1]);
  } else {
    *reinterpret_cast<uint32_t*>(ko) = kw[0];
    *reinterpret_cast<uint32_t*>(vo) = vw[0];
  }
  if (range_hit) atomicOr(p.status, JATTN_DEV_RANGE);
}

template <int D, int OUT>
cudaError_t launch_rope_t(const RopeParams& p, cudaStream_t st) {
  constexpr int NT = D / 8 * kTok / kTokPerThread;
  dim3 grid(p.nblk, p.B);
  const bool repair = OUT == kOutE4M3 && p.score != nullptr;
  if constexpr (OUT == kOutF16) {
    if (p.hp) {
      if (p.norm_w != nullptr) rope_qkv_kernel<D, OUT, true, false, true><<<grid, NT, 0, st>>>(p);
      else rope_qkv_kernel<D, OUT, false, false, true><<<grid, NT, 0, st>>>(p);
      return cudaGetLastError();
    }
  }
  if (repair) {
    if (p.norm_w != nullptr) rope_qkv_kernel<D, OUT, true, OUT == kOutE4M3, false><<<grid, NT, 0, st>>>(p);
    else rope_qkv_kernel<D, OUT, false, OUT == kOutE4M3, false><<<grid, NT, 0, st>>>(p);
  } else {
    if (p.norm_w != nullptr) rope_qkv_kernel<D, OUT, true, false, false><<<grid, NT, 0, st>>>(p);
    else rope_qkv_kernel<D, OUT, false, false, false><<<grid, NT, 0, st>>>(p);
  }
  return cudaGetLastError();
}

template <int D, bool BF>
cudaError_t launch_quant_t(const QuantParams& p, cudaStream_t st) {
  constexpr int NT = D / 8 * kTok / kTokPerThread;
  dim3 grid(p.nblk, p.BH);
  quant_fp8_kernel<D, BF><<<grid, NT, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope_qkv(const RopeParams& p, int out_kind, cudaStream_t st) {
  if (p.d == 128) {
    if (out_kind == 0) return launch_rope_t<128, kOutF16>(p, st);
    if (out_kind == 1) return launch_rope_t<128, kOutBF16>(p, st);
    return launch_rope_t<128, kOutE4M3>(p, st);
  }
  if (out_kind == 0) return launch_rope_t<64, kOutF16>(p, st);
  if (out_kind == 1) return launch_rope_t<64, kOutBF16>(p, st);
  return launch_rope_t<64, kOutE4M3>(p, st);
}

cudaError_t launch_repair_gather(const GatherParams& p, cudaStream_t st) {
  if (p.n <= 0) return cudaSuccess;
  dim3 grid((p.n + 7) / 8, p.B * p.H);
  if (p.d == 128) repair_gather_kernel<128><<<grid, 256, 0, st>>>(p);
  else repair_gather_kernel<64><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const QuantParams& p, bool in_bf16, cudaStream_t st) {
  if (p.d == 128) return in_bf16 ? launch_quant_t<128, true>(p, st) : launch_quant_t<128, false>(p, st);
  return in_bf16 ? launch_quant_t<64, true>(p, st) : launch_quant_t<64, false>(p, st);
}

}  // namespace jattn
