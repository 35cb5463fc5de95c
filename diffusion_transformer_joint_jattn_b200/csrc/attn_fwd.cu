// Joint-attention forward on sm_100a: O = softmax(Q K^T * scale) V over the
// whole joint sequence, with 16-bit (fp16 / bf16) or e4m3 operands.
//
// Method ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA
// Blackwell GPUs", section "Quantized and sparse attention"): dense attention
// over the joined text / image / reference tokens, in a BF16 path and an FP8
// path with FP8 query/key and FP8 value.  The page names library kernels only;
// this kernel is written for B200 from the definition.
//
// One CTA computes one 128-row query tile of one (batch, head):
//   warp 4      TMA producer: Q once, then K_j and V_j tiles into smem rings
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T into TMEM (two S
//               buffers), then O += P_{j-1} V_{j-1} with P read from TMEM
//   warps 0..3  softmax: one thread per query row (= TMEM lane); online
//               softmax with a lazy rescale (O and l are rescaled only when
//               the running max grows by more than 2^8), P written back to
//               TMEM as fp16 / e4m3; epilogue O / l -> bf16 [B, S, H, d].
// Accumulators live in TMEM: S0 [0,128), S1 [128,256), O [256, 256+d),
// P [384, 448).  Every wait is bounded (see ptx_sm100.cuh).
#include <cstdint>
#include <cuda_runtime.h>

#include "jattn.h"
#include "jattn_internal.h"
#include "ptx_sm100.cuh"

namespace jattn {

namespace {

constexpr int BM = 128;              // query rows per CTA
constexpr int BN = 128;              // keys per tile
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP = 384;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: P <= 2^8 before rescale

template <int D, bool FP8>
struct Cfg {
  static constexpr int ES = FP8 ? 1 : 2;              // element bytes
  static constexpr int RB = D * ES;                   // row bytes
  static constexpr int SWB = RB >= 128 ? 128 : 64;    // swizzle span (bytes)
  static constexpr uint32_t SWMODE = SWB == 128 ? 2u : 4u;
  static constexpr int NBOX = RB / SWB;               // TMA boxes per tile
  static constexpr int BOX_ELEMS = SWB / ES;          // inner box extent (elements)
  static constexpr int BOXB = BM * SWB;               // bytes per box
  static constexpr int TB = BM * RB;                  // bytes per tile
  static constexpr int MK = FP8 ? 32 : 16;            // K per MMA instruction
  static constexpr int QK_STEPS = RB / 32;            // 32 bytes of K per step
  static constexpr int PV_STEPS = BN / MK;
  static constexpr int STAGES = (TB >= 32768) ? 3 : 4;
  static constexpr int SMEM = (1 + 2 * STAGES) * TB + 2048;
  static constexpr int P_COLS = BN * (FP8 ? 1 : 2) / 4;
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full;
  uint64_t o_done;
  uint64_t mma_final;
  uint32_t tmem_base;
  uint32_t abort;
};

// Warp-uniform bounded wait: every lane polls, the whole warp leaves the
// loop together (the tcgen05.ld/st that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    const bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((i & 63u) == 63u) {
      int stop = 0;
      if (lane_id() == 0) {
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        if (*ctl.abort) stop = 1;
        else if (now - t0 > ctl.limit_ns) {
          atomicOr(ctl.status, JATTN_DEV_TIMEOUT);
          *ctl.abort = 1u;
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
}

// Wait that ignores the abort flag (used only to drain in-flight async work
// before the CTA exits); still time-limited.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      atomicOr(ctl.status, JATTN_DEV_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// KIND: 0 = fp16 operands, 1 = bf16 operands, 2 = e4m3 operands.
template <int D, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  constexpr bool FP8 = KIND == 2;
  constexpr uint32_t in_fmt = KIND == 1 ? 1u : 0u;   // f16 / bf16 (kind::f16); e4m3 (kind::f8f6f4)
  using C = Cfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::TB;
  uint8_t* sV = sK + C::STAGES * C::TB;
  Bars* bar = reinterpret_cast<Bars*>(sV + C::STAGES * C::TB);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.H, h = bh % p.H;
  const int n_kv = p.n_tiles;

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->s_empty[s], BM);
    }
    mbar_init(&bar->p_full, BM);
    mbar_init(&bar->o_done, 1);
    mbar_init(&bar->mma_final, 1);
    bar->abort = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_alloc(&bar->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const WaitCtl ctl{&bar->abort, p.status, p.timeout_ns};

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar->q_full, C::TB);
      for (int x = 0; x < C::NBOX; ++x)
        tma_load_3d(&tmQ, &bar->q_full, sQ + x * C::BOXB, x * C::BOX_ELEMS, qt * BM, bh);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = ((j / C::STAGES) & 1) ^ 1;
        if (!mbar_wait(&bar->k_empty[s], ph, ctl)) break;
        mbar_arrive_expect_tx(&bar->k_full[s], C::TB);
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_3d(&tmK, &bar->k_full[s], sK + s * C::TB + x * C::BOXB, x * C::BOX_ELEMS, j * BN, bh);
        if (!mbar_wait(&bar->v_empty[s], ph, ctl)) { issued = 2 * j + 1; break; }
        mbar_arrive_expect_tx(&bar->v_full[s], C::TB);
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_3d(&tmV, &bar->v_full[s], sV + s * C::TB + x * C::BOXB, x * C::BOX_ELEMS, j * BN, bh);
        issued = 2 * j + 2;
      }
      // Drain: every load issued must have landed before the CTA may exit.
      drain_wait(&bar->q_full, 0, ctl);
      const int nk = (issued + 1) / 2, nv = issued / 2;
      for (int s = 0; s < C::STAGES; ++s) {
        if (s < nk) drain_wait(&bar->k_full[s], ((nk - 1 - s) / C::STAGES) & 1, ctl);
        if (s < nv) drain_wait(&bar->v_full[s], ((nv - 1 - s) / C::STAGES) & 1, ctl);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = instr_desc(in_fmt, in_fmt, 0, BM, BN);
      const uint32_t idesc_pv = instr_desc(in_fmt, in_fmt, 1, BM, D);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = mbar_wait(&bar->q_full, 0, ctl);
      bool any_mma = false;
      auto issue_pv = [&](int i) -> bool {
        const int s = i % C::STAGES;
        if (!mbar_wait(&bar->p_full, i & 1, ctl)) return false;
        if (!mbar_wait(&bar->v_full[s], (i / C::STAGES) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t vbase = sVa + s * C::TB;
#pragma unroll
        for (int kk = 0; kk < C::PV_STEPS; ++kk) {
          const uint64_t bdesc = smem_desc(vbase + kk * C::MK * C::SWB, C::BOXB, 8 * C::SWB, C::SWMODE);
          if constexpr (FP8) mma_f8_ts(tmem + kColO, tmem + kColP + kk * 8, bdesc, idesc_pv, (i > 0 || kk > 0));
          else mma_f16_ts(tmem + kColO, tmem + kColP + kk * 8, bdesc, idesc_pv, (i > 0 || kk > 0));
        }
        mma_commit(&bar->v_empty[s]);
        mma_commit(&bar->o_done);
        return true;
      };
      if (ok) {
        tc_fence_after();
        for (int j = 0; j < n_kv && ok; ++j) {
          const int s = j % C::STAGES, sb = j & 1;
          ok = mbar_wait(&bar->k_full[s], (j / C::STAGES) & 1, ctl) &&
               mbar_wait(&bar->s_empty[sb], ((j >> 1) & 1) ^ 1, ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kbase = sKa + s * C::TB;
          const uint32_t d_s = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
          for (int kk = 0; kk < C::QK_STEPS; ++kk) {
            const uint32_t off = (kk * 32) / C::SWB * C::BOXB + (kk * 32) % C::SWB;
            const uint64_t adesc = smem_desc(sQa + off, 16, 8 * C::SWB, C::SWMODE);
            const uint64_t bdesc = smem_desc(kbase + off, 16, 8 * C::SWB, C::SWMODE);
            if constexpr (FP8) mma_f8_ss(d_s, adesc, bdesc, idesc_qk, kk > 0);
            else mma_f16_ss(d_s, adesc, bdesc, idesc_qk, kk > 0);
          }
          any_mma = true;
          mma_commit(&bar->s_full[sb]);
          mma_commit(&bar->k_empty[s]);
          if (j > 0) ok = issue_pv(j - 1);
        }
        if (ok) issue_pv(n_kv - 1);
      }
      if (any_mma) {
        mma_commit(&bar->mma_final);
        drain_wait(&bar->mma_final, 0, ctl);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = warp * 32 + lane;                 // TMEM lane == query row
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    const int q_row = qt * BM + row;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;

    float sq = 1.f, max_sv = 1.f;
    const float* sc_k = nullptr;
    const float* sc_v = nullptr;
    if constexpr (FP8) {
      const size_t nb = static_cast<size_t>(p.n_tiles);
      const size_t bhn = static_cast<size_t>(bh) * nb;
      const size_t plane = static_cast<size_t>(p.B) * p.H * nb;
      sq = p.scales[bhn + qt];
      sc_k = p.scales + plane + bhn;
      sc_v = p.scales + 2 * plane + bhn;
      float mv = 0.f;
      for (int j = lane; j < n_kv; j += 32) mv = fmaxf(mv, sc_v[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
      max_sv = mv > 0.f ? mv : 1.f;
    }
    // FP8: P is stored as p * (s_v,j / max s_v) * 448 / 2^8 so that it never
    // exceeds the e4m3 range while p <= 2^8.
    const float p8_log2 = 8.8073549220576042f - kRescaleThreshold;   // log2(448) - 8

    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      ok = warp_wait(&bar->s_full[sb], (j >> 1) & 1, ctl);
      if (!ok) break;
      __syncwarp();
      tc_fence_after();
      float v[BN];
      {
        uint32_t r[32];
        const uint32_t ts = tmem + lane_base + (sb ? kColS1 : kColS0);
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          tmem_ld32(ts + c * 32, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[c * 32 + e] = __uint_as_float(r[e]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar->s_empty[sb]);

      float c_j = sl2, bias = 0.f;
      if constexpr (FP8) {
        c_j = sl2 * sq * sc_k[j];
        bias = __log2f(sc_v[j] / max_sv) + p8_log2;
      }
      const int valid = p.S - j * BN;
      if (valid < BN) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e >= valid) v[e] = -INFINITY;
      }
      float mx = v[0];
#pragma unroll
      for (int e = 1; e < BN; ++e) mx = fmaxf(mx, v[e]);
      mx *= c_j;
      const float m_new = fmaxf(m_run, mx);
      float alpha = 1.f;
      const bool resc = (m_new - m_run) > kRescaleThreshold;
      if (resc) {
        alpha = ex2_approx(m_run - m_new);
        m_run = m_new;
        l_run *= alpha;
      }
      const float neg_m = bias - m_run;
      float ls = 0.f;
      uint32_t pk[C::P_COLS];
      if constexpr (FP8) {
#pragma unroll
        for (int c = 0; c < C::P_COLS; ++c) {
          const float p0 = ex2_approx(fmaf(v[4 * c + 0], c_j, neg_m));
          const float p1 = ex2_approx(fmaf(v[4 * c + 1], c_j, neg_m));
          const float p2 = ex2_approx(fmaf(v[4 * c + 2], c_j, neg_m));
          const float p3 = ex2_approx(fmaf(v[4 * c + 3], c_j, neg_m));
          ls += (p0 + p1) + (p2 + p3);
          pk[c] = pack_e4m3x4(p0, p1, p2, p3);
        }
        ls *= ex2_approx(-bias);
      } else {
#pragma unroll
        for (int c = 0; c < C::P_COLS; ++c) {
          const float p0 = ex2_approx(fmaf(v[2 * c + 0], c_j, neg_m));
          const float p1 = ex2_approx(fmaf(v[2 * c + 1], c_j, neg_m));
          ls += p0 + p1;
          pk[c] = KIND == 1 ? pack_bf16x2(p0, p1) : pack_f16x2(p0, p1);
        }
      }
      l_run += ls;

      if (j > 0) {
        // P_{j-1} consumed and O final up to tile j-1 before P_j / rescale.
        ok = warp_wait(&bar->o_done, (j - 1) & 1, ctl);
        if (!ok) break;
        __syncwarp();
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            const uint32_t to = tmem + lane_base + kColO + c * 32;
            tmem_ld32(to, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(to, r);
          }
        }
      }
      __syncwarp();
      {
        const uint32_t tp = tmem + lane_base + kColP;
#pragma unroll
        for (int c = 0; c < C::P_COLS / 32; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = pk[c * 32 + e];
          tmem_st32(tp + c * 32, r);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar->p_full);
    }

    if (ok) ok = warp_wait(&bar->o_done, (n_kv - 1) & 1, ctl);
    if (ok) {
      __syncwarp();
      tc_fence_after();
      float out_scale = 1.f / l_run;
      if constexpr (FP8) out_scale *= max_sv * ex2_approx(-p8_log2);
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.S + q_row) * p.H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(tmem + lane_base + kColO + c * 32, r);
        if (q_row < p.S) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * out_scale,
                                                      __uint_as_float(r[2 * e + 1]) * out_scale);
            w[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      if (p.lse != nullptr && q_row < p.S)
        p.lse[static_cast<size_t>(bh) * p.S + q_row] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int KIND>
cudaError_t launch_t(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     cudaStream_t st) {
  using C = Cfg<D, KIND == 2>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  auto kern = attn_fwd_kernel<D, KIND>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_tiles, p.B * p.H);
  kern<<<grid, kThreads, C::SMEM, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

// Bounded-wait self test: waits on a barrier nobody arrives on.
__global__ void selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const WaitCtl ctl{&abort_flag, status, limit_ns};
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, ctl);
  __syncthreads();
}

}  // namespace

cudaError_t launch_fwd_f16(const FwdParams& p, int d, bool in_bf16, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  if (in_bf16) return d == 128 ? launch_t<128, 1>(p, tq, tk, tv, st) : launch_t<64, 1>(p, tq, tk, tv, st);
  return d == 128 ? launch_t<128, 0>(p, tq, tk, tv, st) : launch_t<64, 0>(p, tq, tk, tv, st);
}

cudaError_t launch_fwd_fp8(const FwdParams& p, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, cudaStream_t st) {
  return d == 128 ? launch_t<128, 2>(p, tq, tk, tv, st) : launch_t<64, 2>(p, tq, tk, tv, st);
}

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace jattn
