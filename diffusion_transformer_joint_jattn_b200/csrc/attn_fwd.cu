// Joint-attention forward on sm_100a: O = softmax(Q K^T * scale) V over the
// whole joint sequence, with 16-bit (fp16 / bf16) or e4m3 operands.
//
// Method ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA
// Blackwell GPUs", section "Quantized and sparse attention"): dense attention
// over the joined text / image / reference tokens, in a BF16 path and an FP8
// path with FP8 query/key and FP8 value.  The page names library kernels only;
// this kernel is written for B200 from the definition.
//
// Work items (batch * head, pair of query tiles): a CTA walks items with a
// stride of the grid size; barrier phases and ring positions run on across
// items, so the next item's Q load and first Q.K^T overlap the current
// item's epilogue.  The grid is one CTA per item, or one per SM when items
// walk only a few key tiles.  Per item the CTA computes two 128-row query
// tiles (t = 0, 1) of one (batch, head):
//   warps 0..3  softmax of tile 0, warps 4..7 softmax of tile 1: one thread
//               per query row (= TMEM lane), online softmax with a lazy
//               rescale (O and l are rescaled only when the running max grows
//               by more than 2^15 -- 2^8 with e4m3 P), P written back into
//               the tile's S columns;
//               epilogue O / l -> bf16 [B, S, H, d].
//   warp 8      MMA issuer (one thread): S_t = Q_t K_j^T, O_t += P_t V_j.
//               Issue order PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1): each
//               tile's softmax overlaps the other tile's tensor work.  With
//               e4m3 operands P is handed over in two halves of 64 keys, so
//               the first half's P.V overlaps the second half's softmax.
//   warp 9      TMA producer: the item's Q tiles (once the previous item's
//               Q.K^T are done), K_j / V_j into smem rings.
//   (warps 10, 11 idle: they complete the third warpgroup.)
// The block starts at 168 registers per thread (384 x 168 = 64512); the
// MMA/TMA warpgroup then releases registers and the two softmax warpgroups
// grow (224 / 56 for e4m3 operands, 216 / 72 for the 16-bit instances at
// d = 128, 208 / 88 at d = 64; 2 x 128 x softmax + 128 x other = 64512).
// TMEM: S_0 [0,128), S_1 [128,256), O_0 [256, 256+d), O_1 [384, 384+d).
// Because the tensor pipe runs one thread's MMAs in order, the commit that
// signals S_t(j) also proves PV_t(j-1) finished: O_t is stable for the
// rescale, and P_t(j-1) has been consumed before S_t(j) overwrites it.
// Every wait is bounded (see ptx_sm100.cuh).
#include <cstdint>
#include <cuda_runtime.h>

#include "jattn.h"
#include "jattn_internal.h"
#include "ptx_sm100.cuh"

namespace jattn {

namespace {

constexpr int BM = 128;              // query rows per tile
constexpr int NQ = 2;                // query tiles per CTA
constexpr int BN = 128;              // keys per tile
constexpr int kMmaWarp = 8;
constexpr int kProducerWarp = 9;
constexpr int kThreads = 384;
// Register split after setmaxnreg (multiples of 8, together exactly the
// 384 x 168 the block launches with): ptxas allocates each role's code within
// its share, and a spill in the single MMA-issuing thread sits on the
// S -> P -> MMA chain, so each instance gets the split that leaves its
// softmax and its MMA / TMA code spill-free at d = 128 (checked with
// -Xptxas -v).
template <int D, int KIND, bool HP, bool SPARSE>
__host__ __device__ constexpr uint32_t regs_softmax() {
  return KIND == 2 ? 224u : (D == 128 ? 216u : 208u);
}
template <int D, int KIND, bool HP, bool SPARSE>
__host__ __device__ constexpr uint32_t regs_other() {
  return (kThreads * 168u - 2u * 128u * regs_softmax<D, KIND, HP, SPARSE>()) / 128u;
}
constexpr uint32_t kTmemCols = 512;
// Launch one persistent CTA per SM when every item walks at most this many
// key tiles (the 16-bit pass over a few repaired keys); otherwise one CTA per
// item, which measured at least as fast for long key walks.
constexpr int kPersistentMaxKv = 4;
// Lazy rescale: O and l are rescaled only when a row's running max grows by
// more than this many log2 units, so P <= 2^threshold in between.  16-bit P
// has room for 2^15 (fewer rescales); e4m3 P keeps 2^8 so that P * 448 / 2^8
// stays in range without pushing small probabilities into subnormals.
constexpr float kRescaleThreshold16 = 15.0f;
constexpr float kRescaleThreshold8 = 8.0f;

__host__ __device__ constexpr uint32_t col_s(int t) { return static_cast<uint32_t>(t) * 128u; }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + static_cast<uint32_t>(t) * 128u; }

// HP: the high-precision 16-bit instance, which also stages one correction
// tile (128 rows x 16 fp16 = 32 bytes, 32-byte swizzle) per query tile and
// per K stage.
template <int D, bool FP8, bool HP = false>
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
  static constexpr int KS = TB >= 32768 ? (HP ? 2 : 3) : 4;   // K ring stages
  static constexpr int VS = TB >= 32768 ? 2 : 4;      // V ring stages
  static constexpr int CT = HP ? BM * 32 : 0;         // correction tile bytes
  static constexpr int SMEM = (NQ + KS + VS) * TB + (NQ + KS) * CT + 2048;
};

struct __align__(8) Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t s_full[NQ], p_full[NQ], o_final[NQ];
  uint64_t p_half[NQ];            // FP8: P of the tile's first 64 keys is in TMEM
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
// The value itself, hidden from the compiler's loop-invariant analysis.
__device__ __forceinline__ uint32_t opaque(uint32_t x) {
  uint32_t y;
  asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// KIND: 0 = fp16 operands, 1 = bf16 operands, 2 = e4m3 operands.
// HP (KIND 0 only): the high-precision 16-bit path -- per-block power-of-two
// range scales of Q, K and V folded in like the e4m3 block scales, and each
// logit tile completed by Qc . Kc^T over the correction tiles (tmQc, tmKc).
// SPARSE: walk the CTA's key-tile list (block-sparse attention) instead of
// every key tile; a separate instance so the dense ones carry no list state.
template <int D, int KIND, bool HP, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQc,
                const __grid_constant__ CUtensorMap tmKc, const FwdParams p) {
  constexpr bool FP8 = KIND == 2;
  constexpr bool SCALED = FP8 || HP;                   // per-block scales of Q, K and V
  static_assert(!HP || KIND == 0, "the high-precision path has fp16 operands");
  constexpr uint32_t in_fmt = KIND == 1 ? 1u : 0u;   // f16 / bf16 (kind::f16); e4m3 (kind::f8f6f4)
  using C = Cfg<D, FP8, HP>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms.
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);
  uint8_t* sQ = smem;                                  // NQ tiles
  uint8_t* sK = sQ + NQ * C::TB;
  uint8_t* sV = sK + C::KS * C::TB;
  uint8_t* sQc = sV + C::VS * C::TB;                   // HP: NQ correction tiles, then KS
  uint8_t* sKc = sQc + NQ * C::CT;
  Bars* bar = reinterpret_cast<Bars*>(sKc + C::KS * C::CT);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Work items: (batch * head, pair of query tiles), pairs fastest; this CTA
  // takes items blockIdx.x, blockIdx.x + gridDim.x, ...  Every barrier's
  // phase runs on across items (global step and tile counters).
  const int n_qp = (p.n_tiles + NQ - 1) / NQ;
  const int n_items = n_qp * p.B * p.H;
  // Key tiles of an item: all n_kv in order, or (block-sparse) the first
  // kv_count entries of its kv_list row.
  auto item_kv = [&](int it) {
    if constexpr (SPARSE) return p.kv_count[it];
    else return p.n_kv;
  };
  auto kv_tile = [&](int it, int j) {
    if constexpr (SPARSE) return __ldg(p.kv_list + static_cast<size_t>(it) * p.n_kv + j);
    else return j;
  };

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    for (int s = 0; s < C::KS; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
    }
    for (int s = 0; s < C::VS; ++s) {
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(&bar->s_full[t], 1);
      mbar_init(&bar->p_full[t], BM);
      mbar_init(&bar->p_half[t], BM);
      mbar_init(&bar->o_final[t], 1);
    }
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
  if (warp >= 8) {
    // Third warpgroup: producer, MMA issuer and two idle warps.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(regs_other<D, KIND, HP, SPARSE>()));
    if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if constexpr (HP) {
        tma_prefetch_desc(&tmQc);
        tma_prefetch_desc(&tmKc);
      }
      int nq = 0, nk = 0, nv = 0;                   // loads issued: Q pairs, K tiles, V tiles
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const int bh = it / n_qp, qp = it % n_qp;
        const int n_kv = item_kv(it);
        // the Q buffer is free once the previous item's Q.K^T are done
        if (nq > 0 && !mbar_wait(&bar->q_empty, (nq - 1) & 1, ctl)) break;
        mbar_arrive_expect_tx(&bar->q_full, NQ * (C::TB + C::CT));
        for (int t = 0; t < NQ; ++t) {
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_3d(&tmQ, &bar->q_full, sQ + t * C::TB + x * C::BOXB, x * C::BOX_ELEMS, (qp * NQ + t) * BM, bh);
          if constexpr (HP) tma_load_3d(&tmQc, &bar->q_full, sQc + t * C::CT, 0, (qp * NQ + t) * BM, bh);
        }
        ++nq;
        for (int j = 0; j < n_kv; ++j) {
          const int ks = nk % C::KS;
          if (!mbar_wait(&bar->k_empty[ks], ((nk / C::KS) & 1) ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&bar->k_full[ks], C::TB + C::CT);
          const int kt = kv_tile(it, j);
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_3d(&tmK, &bar->k_full[ks], sK + ks * C::TB + x * C::BOXB, x * C::BOX_ELEMS, kt * BN, bh);
          if constexpr (HP) tma_load_3d(&tmKc, &bar->k_full[ks], sKc + ks * C::CT, 0, kt * BN, bh);
          ++nk;
          const int vs = nv % C::VS;
          if (!mbar_wait(&bar->v_empty[vs], ((nv / C::VS) & 1) ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&bar->v_full[vs], C::TB);
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_3d(&tmV, &bar->v_full[vs], sV + vs * C::TB + x * C::BOXB, x * C::BOX_ELEMS, kt * BN, bh);
          ++nv;
        }
      }
      // Drain: every load issued must have landed before the CTA may exit.
      if (nq > 0) drain_wait(&bar->q_full, (nq - 1) & 1, ctl);
      for (int i = nk > C::KS ? nk - C::KS : 0; i < nk; ++i) drain_wait(&bar->k_full[i % C::KS], (i / C::KS) & 1, ctl);
      for (int i = nv > C::VS ? nv - C::VS : 0; i < nv; ++i) drain_wait(&bar->v_full[i % C::VS], (i / C::VS) & 1, ctl);
    }
    } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = instr_desc(in_fmt, in_fmt, 0, BM, BN);
      const uint32_t idesc_pv = instr_desc(in_fmt, in_fmt, 1, BM, D);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool any_mma = false;
      // e4m3: the tile bases pass through opaque() so that the descriptors
      // are formed next to each MMA instead of being hoisted out of the loops
      // (dozens of 64-bit loop invariants do not fit the 56-register share
      // of this role; the 16-bit instances measured faster without it).
      auto base_of = [](uint32_t x) { return FP8 ? opaque(x) : x; };
      auto issue_qk = [&](int t, int ks) {
        const uint32_t kbase = base_of(sKa + ks * C::TB);
        const uint32_t qbase = base_of(sQa + t * C::TB);
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk) {
          const uint32_t off = (kk * 32) / C::SWB * C::BOXB + (kk * 32) % C::SWB;
          const uint64_t adesc = smem_desc(qbase + off, 16, 8 * C::SWB, C::SWMODE);
          const uint64_t bdesc = smem_desc(kbase + off, 16, 8 * C::SWB, C::SWMODE);
          if constexpr (FP8) mma_f8_ss(tmem + col_s(t), adesc, bdesc, idesc_qk, kk > 0);
          else mma_f16_ss(tmem + col_s(t), adesc, bdesc, idesc_qk, kk > 0);
        }
        if constexpr (HP) {
          // the low-order terms of the selected channels: one 16-deep step
          const uint64_t adesc = smem_desc(smem_u32(sQc) + t * C::CT, 16, 256, kSwizzle32B);
          const uint64_t bdesc = smem_desc(smem_u32(sKc) + ks * C::CT, 16, 256, kSwizzle32B);
          mma_f16_ss(tmem + col_s(t), adesc, bdesc, idesc_qk, 1);
        }
        any_mma = true;
      };
      auto issue_pv = [&](int t, int vs, bool acc, int kk0, int kk1) {
        const uint32_t vbase = base_of(sVa + vs * C::TB);
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk) {
          const uint64_t bdesc = smem_desc(vbase + kk * C::MK * C::SWB, C::BOXB, 8 * C::SWB, C::SWMODE);
          if constexpr (FP8) mma_f8_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8, bdesc, idesc_pv, acc || kk > 0);
          else mma_f16_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8, bdesc, idesc_pv, acc || kk > 0);
        }
      };
      int nq = 0, nk = 0, nv = 0, gs = 0;           // items, K tiles, V tiles, softmax steps so far
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const int n_kv = item_kv(it);
        ok = mbar_wait(&bar->q_full, nq & 1, ctl) && mbar_wait(&bar->k_full[nk % C::KS], (nk / C::KS) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < NQ; ++t) {
          issue_qk(t, nk % C::KS);
          mma_commit(&bar->s_full[t]);
        }
        mma_commit(&bar->k_empty[nk % C::KS]);
        if (n_kv == 1) mma_commit(&bar->q_empty);    // this item's last Q.K^T
        ++nk;
        for (int j = 0; j < n_kv && ok; ++j) {
          const int vs = nv % C::VS;
          const int ks = nk % C::KS;
          const int ph = (gs + j) & 1;                // phase of this step's softmax barriers
          const bool more = j + 1 < n_kv;
          ok = mbar_wait(&bar->v_full[vs], (nv / C::VS) & 1, ctl);
          for (int t = 0; t < NQ && ok; ++t) {
            if constexpr (FP8) {
              // P arrives in two halves: the first half's P.V steps overlap
              // the softmax of the second half.
              ok = mbar_wait(&bar->p_half[t], ph, ctl);
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, vs, j > 0, 0, C::PV_STEPS / 2);
              ok = mbar_wait(&bar->p_full[t], ph, ctl);
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, vs, true, C::PV_STEPS / 2, C::PV_STEPS);
            } else {
              ok = mbar_wait(&bar->p_full[t], ph, ctl);
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, vs, j > 0, 0, C::PV_STEPS);
            }
            if (t == NQ - 1) mma_commit(&bar->v_empty[vs]);
            if (more) {
              if (t == 0) {
                ok = mbar_wait(&bar->k_full[ks], (nk / C::KS) & 1, ctl);
                if (!ok) break;
                tc_fence_after();
              }
              issue_qk(t, ks);
              mma_commit(&bar->s_full[t]);
              if (t == NQ - 1) {
                mma_commit(&bar->k_empty[ks]);
                if (j + 2 == n_kv) mma_commit(&bar->q_empty);   // this item's last Q.K^T
              }
            } else {
              mma_commit(&bar->o_final[t]);
            }
          }
          if (!ok) break;
          ++nv;
          if (more) ++nk;
        }
        gs += n_kv;
        ++nq;
      }
      if (any_mma) {
        mma_commit(&bar->mma_final);
        drain_wait(&bar->mma_final, 0, ctl);
      }
    }
    }
  } else {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(regs_softmax<D, KIND, HP, SPARSE>()));
    const int t = warp >> 2;                          // query tile of this warpgroup
    const int row = (warp & 3) * 32 + lane;           // TMEM lane == row in the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t ts = tmem + lane_base + col_s(t);
    const uint32_t to = tmem + lane_base + col_o(t);
    const float sl2 = p.scale_log2;
    // FP8: P is stored as p * (s_v,j / max s_v) * 448 / 2^8 so that it never
    // exceeds the e4m3 range while p <= 2^8.  HP: as p * (s_v,j / max s_v)
    // (powers of two; at most 2^15 in fp16).
    constexpr float kRescaleThreshold = FP8 ? kRescaleThreshold8 : kRescaleThreshold16;
    const float p8_log2 = FP8 ? 8.8073549220576042f - kRescaleThreshold : 0.f;   // log2(448) - 8
    bool ok = true;
    int gs = 0, nq = 0;                                // softmax steps and items so far
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++nq) {
    const int bh = it / n_qp, qp = it % n_qp;
    const int b = bh / p.H, h = bh % p.H;
    const int n_kv = item_kv(it);
    const int q_row = (qp * NQ + t) * BM + row;
    float m_run = -INFINITY, l_run = 0.f;
    // Merging into a partial result over other keys (lse_prev given: the
    // e4m3 pass of the repair path; the high-precision and block-sparse
    // instances never merge): the row's old output and its LSE are asked
    // into L2 now, so that the epilogue's reads of them do not wait on HBM.
    if (!HP && !SPARSE && p.lse_prev != nullptr && q_row < p.S) {
      const uint8_t* orow0 = reinterpret_cast<const uint8_t*>(p.o + ((static_cast<size_t>(b) * p.S + q_row) * p.H + h) * D);
#pragma unroll
      for (int x = 0; x < D * 2; x += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(orow0 + x));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.lse_prev + static_cast<size_t>(bh) * p.S + q_row));
    }

    float sq = 1.f, max_sv = 1.f;
    bool unit_scales = false;
    const float* sc_k = nullptr;
    const float* sc_v = nullptr;
    if constexpr (SCALED) {
      const size_t nb = static_cast<size_t>(p.n_tiles);
      const size_t bhn = static_cast<size_t>(bh) * nb;
      const size_t plane = static_cast<size_t>(p.B) * p.H * nb;
      sq = p.scales[bhn + min(qp * NQ + t, p.n_tiles - 1)];
      sc_k = p.scales + plane + bhn;
      sc_v = p.scales + 2 * plane + bhn;
      float mv = 0.f;
      bool unit = sq == 1.f;
      for (int j = lane; j < p.n_kv; j += 32) {         // every tile: ratios stay <= 1
        const float a = sc_v[j];
        mv = fmaxf(mv, a);
        if constexpr (HP) unit = unit && a == 1.f && sc_k[j] == 1.f;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
      max_sv = mv > 0.f ? mv : 1.f;
      // HP with every range scale 1 (all ordinary inputs): the tiles need no
      // per-tile scale (uniform across the warp).
      if constexpr (HP) unit_scales = __all_sync(0xffffffffu, unit);
    }
    // The K / V block scales of the next tile are fetched one tile ahead so
    // that their load latency stays off the S -> P chain.
    float sk_nxt = 0.f, sv_nxt = 0.f;
    int kt_cur = n_kv > 0 ? kv_tile(it, 0) : 0;        // key tile of step j
    if constexpr (SCALED) {
      sk_nxt = sc_k[kt_cur];
      sv_nxt = sc_v[kt_cur];
    }

    for (int j = 0; j < n_kv; ++j) {
      const int kt = kt_cur;
      if (j + 1 < n_kv) kt_cur = kv_tile(it, j + 1);
      float c_j = sl2, bias = 0.f;
      if (SCALED && !unit_scales) {
        c_j = sl2 * sq * sk_nxt;
        bias = __log2f(sv_nxt / max_sv) + p8_log2;
        if (j + 1 < n_kv) {
          sk_nxt = sc_k[kt_cur];
          sv_nxt = sc_v[kt_cur];
        }
      }
      // Keys left out of this pass (same for every row of the tile; the e4m3
      // pass of the repair path has them, the high-precision path never
      // does).  The next tile's mask is asked into L1 now so that its load
      // stays off the chain.
      uint4 km = make_uint4(0u, 0u, 0u, 0u);
      if (!HP && p.kmask != nullptr) {
        const uint4* kmrow = reinterpret_cast<const uint4*>(p.kmask) + static_cast<size_t>(bh) * p.n_kv;
        km = __ldg(kmrow + kt);
        if (j + 1 < n_kv) asm volatile("prefetch.global.L1 [%0];" ::"l"(kmrow + kt_cur));
      }
      ok = warp_wait(&bar->s_full[t], (gs + j) & 1, ctl);
      if (!ok) break;
      __syncwarp();
      tc_fence_after();
      float v[BN];
      {
        uint32_t r[BN];
        tmem_ld128(ts, r);
#pragma unroll
        for (int e = 0; e < BN; ++e) v[e] = __uint_as_float(r[e]);
      }

      const int valid = p.S_kv - kt * BN;
      if (valid < BN) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e >= valid) v[e] = -INFINITY;
      }
      // Row max as a ternary tree (128 -> 43 -> 15 -> 5 -> 1): five levels of
      // independent three-input maxima instead of long dependent chains.
      auto row_max = [&]() {
        static_assert(BN == 128, "the tree below covers 128 values");
        float a[43];
#pragma unroll
        for (int i = 0; i < 42; ++i) a[i] = max3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
        a[42] = fmaxf(v[126], v[127]);
        float c[15];
#pragma unroll
        for (int i = 0; i < 14; ++i) c[i] = max3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        c[14] = a[42];
        float e[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) e[i] = max3(c[3 * i], c[3 * i + 1], c[3 * i + 2]);
        return max3(e[0], e[1], fmaxf(e[2], fmaxf(e[3], e[4])));
      };
      float mx_raw = row_max();
      // Keys left out of this pass hold zero codes (their logits are exactly
      // 0, their values 0).  Where the row max is positive they cannot be the
      // max, and their probabilities -- exp2(neg_m) each -- are taken off the
      // row sum below.  Only a warp with a row whose max may be such a zero
      // sets them to -inf one by one.
      float n_left_out = 0.f;
      if ((km.x | km.y | km.z | km.w) != 0u) {
        if (__any_sync(0xffffffffu, !(mx_raw > 0.f))) {
          const uint32_t kw[4] = {km.x, km.y, km.z, km.w};
#pragma unroll
          for (int e = 0; e < BN; ++e)
            if ((kw[e >> 5] >> (e & 31)) & 1u) v[e] = -INFINITY;
          mx_raw = row_max();
        } else {
          n_left_out = static_cast<float>(__popc(km.x) + __popc(km.y) + __popc(km.z) + __popc(km.w));
        }
      }
      const float mx = mx_raw * c_j;
      const float m_new = fmaxf(m_run, mx);
      float alpha = 1.f;
      const bool resc = (m_new - m_run) > kRescaleThreshold;
      if (resc) {
        alpha = ex2_approx(m_run - m_new);
        m_run = m_new;
        l_run *= alpha;
      }
      __syncwarp();
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
        // O_t is stable here: PV_t(j-1) completed before S_t(j) was signalled.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(to + c * 32, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(to + c * 32, r);
        }
      }

      // A row whose keys so far were all left out keeps m = -inf; its
      // probabilities are exp2(-inf) = 0 either way.
      const float neg_m = m_run == -INFINITY ? 0.f : bias - m_run;
      const float2 c2 = make_float2(c_j, c_j);
      const float2 nm2 = make_float2(neg_m, neg_m);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      if constexpr (FP8) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int e = half * 64 + 4 * c;
            const float2 x0 = __ffma2_rn(make_float2(v[e + 0], v[e + 1]), c2, nm2);
            const float2 x1 = __ffma2_rn(make_float2(v[e + 2], v[e + 3]), c2, nm2);
            const float2 e0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
            const float2 e1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
            acc0 = __fadd2_rn(acc0, e0);
            acc1 = __fadd2_rn(acc1, e1);
            pk[c] = pack_e4m3x4(e0.x, e0.y, e1.x, e1.y);
          }
          tmem_st16(ts + half * 16, pk);
          if (half == 0) {
            tc_fence_before();
            mbar_arrive(&bar->p_half[t]);
          }
        }
      } else {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int e = half * 64 + 2 * c;
            const float2 x0 = __ffma2_rn(make_float2(v[e + 0], v[e + 1]), c2, nm2);
            const float2 x1 = __ffma2_rn(make_float2(v[e + 2], v[e + 3]), c2, nm2);
            const float2 e0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
            const float2 e1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
            acc0 = __fadd2_rn(acc0, e0);
            acc1 = __fadd2_rn(acc1, e1);
            pk[c] = KIND == 1 ? pack_bf16x2(e0.x, e0.y) : pack_f16x2(e0.x, e0.y);
            pk[c + 1] = KIND == 1 ? pack_bf16x2(e1.x, e1.y) : pack_f16x2(e1.x, e1.y);
          }
          tmem_st32(ts + half * 32, pk);
        }
      }
      float ls = (acc0.x + acc0.y) + (acc1.x + acc1.y);
      if (n_left_out != 0.f) ls = fmaf(-n_left_out, ex2_approx(neg_m), ls);   // zero-logit keys left out
      if constexpr (SCALED) ls *= ex2_approx(-bias);
      l_run += ls;
      tc_fence_before();
      mbar_arrive(&bar->p_full[t]);
    }

    gs += n_kv;
    if (ok) ok = warp_wait(&bar->o_final[t], nq & 1, ctl);
    if (ok) {
      __syncwarp();
      tc_fence_after();
      float out_scale = 1.f / l_run;
      if constexpr (SCALED) out_scale *= max_sv * ex2_approx(-p8_log2);
      float lse2 = m_run + __log2f(l_run);             // log2 units
      // Merge with a partial result over other keys already in o:
      // O = w_a O_a + w_b O_b with w = 2^(LSE_part - LSE), LSE = log2(2^a + 2^b).
      float w_prev = 0.f;
      if (p.lse_prev != nullptr && q_row < p.S) {
        const float la = p.lse_prev[static_cast<size_t>(bh) * p.S + q_row] * 1.4426950408889634f;
        if (la != -INFINITY) {
          const float mx = fmaxf(la, lse2);
          const float tot = mx + __log2f(ex2_approx(la - mx) + ex2_approx(lse2 - mx));
          w_prev = ex2_approx(la - tot);
          // a row that saw no key in this pass (l = 0) adds nothing
          out_scale = l_run > 0.f ? out_scale * ex2_approx(lse2 - tot) : 0.f;
          lse2 = tot;
        }
      }
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.S + q_row) * p.H + h) * D;
      // Rows start at multiples of 2 * D bytes from o, so a 32-byte aligned o
      // makes every 32-byte piece of every row aligned.
      const bool o_al32 = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(to + c * 32, r);
        if (q_row < p.S) {
          float prev[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) prev[e] = 0.f;
          if (w_prev != 0.f) {
            uint4 pu[4];
            if (o_al32) {
#pragma unroll
              for (int e = 0; e < 2; ++e)
                asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                             : "=r"(pu[2 * e].x), "=r"(pu[2 * e].y), "=r"(pu[2 * e].z), "=r"(pu[2 * e].w),
                               "=r"(pu[2 * e + 1].x), "=r"(pu[2 * e + 1].y), "=r"(pu[2 * e + 1].z),
                               "=r"(pu[2 * e + 1].w)
                             : "l"(orow + c * 32 + e * 16)
                             : "memory");
            } else {
              const uint4* src = reinterpret_cast<const uint4*>(orow + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e) pu[e] = src[e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint4 u = pu[e];
              const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int f = 0; f < 4; ++f) {
                prev[8 * e + 2 * f] = __uint_as_float(uw[f] << 16) * w_prev;
                prev[8 * e + 2 * f + 1] = __uint_as_float(uw[f] & 0xFFFF0000u) * w_prev;
              }
            }
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(fmaf(__uint_as_float(r[2 * e]), out_scale, prev[2 * e]),
                               fmaf(__uint_as_float(r[2 * e + 1]), out_scale, prev[2 * e + 1]));
          if (o_al32) {
            // 256-bit stores: each writes one whole 32-byte sector of the row
#pragma unroll
            for (int e = 0; e < 2; ++e)
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                           ::"l"(orow + c * 32 + e * 16), "r"(w[8 * e]), "r"(w[8 * e + 1]), "r"(w[8 * e + 2]),
                             "r"(w[8 * e + 3]), "r"(w[8 * e + 4]), "r"(w[8 * e + 5]), "r"(w[8 * e + 6]),
                             "r"(w[8 * e + 7])
                           : "memory");
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
      }
      if (p.lse != nullptr && q_row < p.S)
        p.lse[static_cast<size_t>(bh) * p.S + q_row] = lse2 * 0.69314718055994531f;
    }
    }  // items
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Streaming multiprocessors of the current device (looked up once per device).
int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

template <int D, int KIND, bool HP = false, bool SPARSE = false>
cudaError_t launch_t(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tqc, const CUtensorMap& tkc, cudaStream_t st) {
  using C = Cfg<D, KIND == 2, HP>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  auto kern = attn_fwd_kernel<D, KIND, HP, SPARSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  // One CTA per work item, or -- when an item walks only a few key tiles and
  // its set-up and epilogue would dominate -- one persistent CTA per SM.
  const long long items = static_cast<long long>((p.n_tiles + NQ - 1) / NQ) * p.B * p.H;
  const bool persistent = p.n_kv <= kPersistentMaxKv && items > sm_count();
  const int grid = static_cast<int>(persistent ? sm_count() : items);
  kern<<<grid, kThreads, C::SMEM, st>>>(tq, tk, tv, tqc, tkc, p);
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

int fwd_kv_rows() { return BN; }

cudaError_t launch_fwd_f16(const FwdParams& p, int d, bool in_bf16, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  if (p.kv_list != nullptr) {
    if (in_bf16)
      return d == 128 ? launch_t<128, 1, false, true>(p, tq, tk, tv, tq, tk, st)
                      : launch_t<64, 1, false, true>(p, tq, tk, tv, tq, tk, st);
    return d == 128 ? launch_t<128, 0, false, true>(p, tq, tk, tv, tq, tk, st)
                    : launch_t<64, 0, false, true>(p, tq, tk, tv, tq, tk, st);
  }
  if (in_bf16) return d == 128 ? launch_t<128, 1>(p, tq, tk, tv, tq, tk, st) : launch_t<64, 1>(p, tq, tk, tv, tq, tk, st);
  return d == 128 ? launch_t<128, 0>(p, tq, tk, tv, tq, tk, st) : launch_t<64, 0>(p, tq, tk, tv, tq, tk, st);
}

cudaError_t launch_fwd_f16_hp(const FwdParams& p, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const CUtensorMap& tqc, const CUtensorMap& tkc,
                              cudaStream_t st) {
  return d == 128 ? launch_t<128, 0, true>(p, tq, tk, tv, tqc, tkc, st)
                  : launch_t<64, 0, true>(p, tq, tk, tv, tqc, tkc, st);
}

cudaError_t launch_fwd_fp8(const FwdParams& p, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, cudaStream_t st) {
  return d == 128 ? launch_t<128, 2>(p, tq, tk, tv, tq, tk, st) : launch_t<64, 2>(p, tq, tk, tv, tq, tk, st);
}

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace jattn
