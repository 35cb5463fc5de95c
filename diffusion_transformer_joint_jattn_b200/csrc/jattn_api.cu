// C-ABI entry points declared in include/jattn.h: argument validation (all of
// it before any launch), TMA tensor-map encoding, launches on the caller's
// stream, and the per-device status word.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "jattn.h"
#include "jattn_internal.h"

namespace {

// Device errors found by the kernels (JATTN_DEV_* bits).  One word per
// device: every module load gets its own copy.
__device__ uint32_t g_status_word;

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;   // 2 s per pipeline wait
constexpr int kMaxDevices = 64;

uint32_t* status_ptr() {
  static uint32_t* ptrs[kMaxDevices] = {};
  static unsigned long long ctx_ids[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  // Looked up again when the context changed (a cudaDeviceReset in between)
  // or none was current yet (the lookup itself initialises it).
  const unsigned long long ctx = jattn::current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr || ctx == 0 || ctx_ids[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<uint32_t*>(p);
    ctx_ids[dev] = jattn::current_context_id();
  }
  return ptrs[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

jattn_status check_shape(const jattn_shape* s) {
  if (s == nullptr) return JATTN_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->S_txt < 0 || s->S_img < 0 || s->S_ref < 0) return JATTN_ERR_INVALID_ARG;
  const int64_t S = static_cast<int64_t>(s->S_txt) + s->S_img + s->S_ref;
  if (S < 1 || S > (1 << 24)) return JATTN_ERR_INVALID_ARG;
  const int64_t BH = static_cast<int64_t>(s->B) * s->H;
  if (BH > 65535) return JATTN_ERR_INVALID_ARG;                        // grid.y of the per-(b,h) kernels
  if ((S + 2 * JATTN_BLOCK - 1) / (2 * JATTN_BLOCK) * BH > INT32_MAX)   // forward work items (an int)
    return JATTN_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return JATTN_ERR_UNSUPPORTED;
  return JATTN_OK;
}

int total_S(const jattn_shape* s) { return s->S_txt + s->S_img + s->S_ref; }
int n_blocks(int S) { return (S + JATTN_BLOCK - 1) / JATTN_BLOCK; }

// [BH][S][d] tensor map; boxes of (one swizzle span of d) x box_rows rows.
jattn_status make_map(CUtensorMap* m, const void* base, int BH, int S, int d, int elem_bytes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return JATTN_ERR_CUDA;
  const int row_bytes = d * elem_bytes;
  const int sw_bytes = row_bytes >= 128 ? 128 : 64;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(row_bytes) * S};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(sw_bytes / elem_bytes), static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUtensorMapSwizzle sw = sw_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? JATTN_OK : JATTN_ERR_CUDA;
}

// [BH][S][16] fp16 correction rows; boxes of 16 x box_rows, 32-byte swizzle.
jattn_status make_map_corr(CUtensorMap* m, const void* base, int BH, int S, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return JATTN_ERR_CUDA;
  const int row_bytes = jattn::kCorrCols * 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(jattn::kCorrCols), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(row_bytes) * S};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(jattn::kCorrCols), static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? JATTN_OK : JATTN_ERR_CUDA;
}

float resolve_scale(float softmax_scale, int d) {
  return softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
}

jattn_status rope_common(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img, const void* qkv_ref,
                         const int32_t* pos, float theta, const int32_t split[3], const float* norm_w, float eps,
                         jattn_dtype out_dtype, void* q, void* k, void* v, float* scales, void* stream,
                         void* q16 = nullptr, float* score = nullptr, float* pair_stat = nullptr,
                         float* norm_r = nullptr) {
  jattn_status st = check_shape(shape);
  if (st != JATTN_OK) return st;
  if (split == nullptr || pos == nullptr || q == nullptr || k == nullptr || v == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!(theta > 0.f) || !std::isfinite(theta)) return JATTN_ERR_INVALID_ARG;
  if (split[0] < 0 || split[1] < 0 || split[2] < 0 || (split[0] | split[1] | split[2]) & 1 ||
      split[0] + split[1] + split[2] != shape->d)
    return JATTN_ERR_INVALID_ARG;
  const void* parts[3] = {qkv_txt, qkv_img, qkv_ref};
  const int lens[3] = {shape->S_txt, shape->S_img, shape->S_ref};
  for (int i = 0; i < 3; ++i) {
    if (lens[i] > 0 && parts[i] == nullptr) return JATTN_ERR_INVALID_ARG;
    if (lens[i] > 0 && !aligned16(parts[i])) return JATTN_ERR_ALIGNMENT;
  }
  if (out_dtype != JATTN_BF16 && out_dtype != JATTN_FP16 && out_dtype != JATTN_E4M3) return JATTN_ERR_UNSUPPORTED;
  if (out_dtype == JATTN_E4M3 && scales == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(pos)) return JATTN_ERR_ALIGNMENT;
  if (norm_w != nullptr && !aligned16(norm_w)) return JATTN_ERR_ALIGNMENT;

  jattn::RopeParams p{};
  for (int i = 0; i < 3; ++i) {
    p.src[i] = static_cast<const __nv_bfloat16*>(parts[i]);
    p.S_part[i] = lens[i];
    p.split[i] = split[i];
  }
  p.B = shape->B;
  p.H = shape->H;
  p.S = total_S(shape);
  p.d = shape->d;
  p.nblk = n_blocks(p.S);
  p.pos = pos;
  p.theta = static_cast<double>(theta);
  p.rope = jattn::make_rope_table(p.theta, p.split, p.d);
  p.dst[0] = q;
  p.dst[1] = k;
  p.dst[2] = v;
  p.scales = scales;
  p.norm_w = norm_w;
  p.eps = eps;
  p.q16 = q16;
  p.score = score;
  p.hp = pair_stat != nullptr ? 1 : 0;
  p.pair_stat = pair_stat;
  p.norm_r = norm_r;
  p.status = status_ptr();
  if (p.status == nullptr) return JATTN_ERR_CUDA;
  const int kind = out_dtype == JATTN_FP16 ? 0 : (out_dtype == JATTN_BF16 ? 1 : 2);
  return jattn::launch_rope_qkv(p, kind, static_cast<cudaStream_t>(stream)) == cudaSuccess ? JATTN_OK
                                                                                          : JATTN_ERR_CUDA;
}

int repair_n(const jattn_shape* shape, float rho) {
  const int S = total_S(shape);
  if (!(rho > 0.f)) return 0;
  const double x = std::ceil(static_cast<double>(rho) * S - 1e-3);
  return x <= 0.0 ? 0 : (x >= S ? S : static_cast<int>(x));
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Scratch of the high-precision prologue: pair statistics, selected pairs,
// RMSNorm row factors (each segment 256-byte aligned).
struct HpLayout {
  size_t pair_stat, sel, norm_r, total;
};

HpLayout hp_layout(const jattn_shape* shape) {
  const size_t BH = static_cast<size_t>(shape->B) * shape->H;
  const size_t S = total_S(shape), d = shape->d, nb = n_blocks(static_cast<int>(S));
  HpLayout L{};
  size_t off = 0;
  auto seg = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
  L.pair_stat = seg(2 * BH * nb * (d / 2) * 4);
  L.sel = seg(BH * jattn::kCorrPairs * 4);
  L.norm_r = seg(2 * BH * S * 4);
  L.total = off;
  return L;
}

// Workspace segments, each 256-byte aligned, in this order.
struct RepairLayout {
  size_t q8, k8, v8, scales, q16, score, idx, kmask, kr, vr, lse, total;
};

RepairLayout repair_layout(const jattn_shape* shape, int n) {
  const size_t BH = static_cast<size_t>(shape->B) * shape->H;
  const size_t S = total_S(shape), d = shape->d, nb = n_blocks(static_cast<int>(S));
  RepairLayout L{};
  size_t off = 0;
  auto seg = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
  L.q8 = seg(BH * S * d);
  L.k8 = seg(BH * S * d);
  L.v8 = seg(BH * S * d);
  L.scales = seg(3 * BH * nb * 4);
  L.q16 = seg(BH * S * d * 2);
  L.score = seg(2 * BH * S * 4);
  L.idx = seg(BH * n * 4);
  L.kmask = seg(BH * nb * 16);
  L.kr = seg(BH * n * d * 2);
  L.vr = seg(BH * n * d * 2);
  L.lse = seg(BH * S * 4);
  L.total = off;
  return L;
}

}  // namespace

namespace jattn {

unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

}  // namespace jattn

extern "C" {

jattn_status jattn_rope_qkv(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                            const void* qkv_ref, const int32_t* pos, float theta, const int32_t split[3],
                            jattn_dtype out_dtype, void* q, void* k, void* v, float* scales, void* stream) {
  return rope_common(shape, qkv_txt, qkv_img, qkv_ref, pos, theta, split, nullptr, 0.f, out_dtype, q, k, v, scales,
                     stream);
}

jattn_status jattn_rope_qkv_norm(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                                 const void* qkv_ref, const int32_t* pos, float theta, const int32_t split[3],
                                 const float* norm_w, float eps, jattn_dtype out_dtype, void* q, void* k,
                                 void* v, float* scales, void* stream) {
  if (norm_w == nullptr || !(eps > 0.f) || !std::isfinite(eps)) return JATTN_ERR_INVALID_ARG;
  return rope_common(shape, qkv_txt, qkv_img, qkv_ref, pos, theta, split, norm_w, eps, out_dtype, q, k, v, scales,
                     stream);
}

jattn_status jattn_quant_fp8(const jattn_shape* shape, jattn_dtype in_dtype, const void* x, void* x8,
                             float* scales, void* stream) {
  jattn_status st = check_shape(shape);
  if (st != JATTN_OK) return st;
  if (x == nullptr || x8 == nullptr || scales == nullptr) return JATTN_ERR_INVALID_ARG;
  if (in_dtype != JATTN_BF16 && in_dtype != JATTN_FP16) return JATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x8)) return JATTN_ERR_ALIGNMENT;
  jattn::QuantParams p{};
  p.x = x;
  p.x8 = x8;
  p.scales = scales;
  p.BH = shape->B * shape->H;
  p.S = total_S(shape);
  p.d = shape->d;
  p.nblk = n_blocks(p.S);
  return jattn::launch_quant_fp8(p, in_dtype == JATTN_BF16, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? JATTN_OK
             : JATTN_ERR_CUDA;
}

static jattn_status fwd_common(const jattn_shape* shape, const void* q, const void* k, const void* v, void* o,
                               float* lse, float softmax_scale, jattn::FwdParams& p) {
  jattn_status st = check_shape(shape);
  if (st != JATTN_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return JATTN_ERR_ALIGNMENT;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return JATTN_ERR_ALIGNMENT;
  p.B = shape->B;
  p.H = shape->H;
  p.S = total_S(shape);
  p.n_tiles = n_blocks(p.S);
  p.S_kv = p.S;
  p.n_kv = p.n_tiles;
  p.kmask = nullptr;
  p.lse_prev = nullptr;
  p.scale_log2 = resolve_scale(softmax_scale, shape->d) * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = status_ptr();
  p.timeout_ns = kDefaultTimeoutNs;
  p.trace = nullptr;
#ifdef JATTN_TRACE
  if (const char* env = std::getenv("JATTN_TRACE_PTR")) p.trace = reinterpret_cast<long long*>(std::strtoull(env, nullptr, 0));
#endif
  if (p.status == nullptr) return JATTN_ERR_CUDA;
  return JATTN_OK;
}

jattn_status jattn_fwd_bf16(const jattn_shape* shape, jattn_dtype in_dtype, const void* q, const void* k,
                            const void* v, void* o, float* lse, float softmax_scale, void* stream) {
  if (in_dtype != JATTN_BF16 && in_dtype != JATTN_FP16) return JATTN_ERR_UNSUPPORTED;
  jattn::FwdParams p{};
  jattn_status st = fwd_common(shape, q, k, v, o, lse, softmax_scale, p);
  if (st != JATTN_OK) return st;
  CUtensorMap tq, tk, tv;
  const int BH = p.B * p.H;
  const int kv_rows = jattn::fwd_kv_rows();
  if ((st = make_map(&tq, q, BH, p.S, shape->d, 2, JATTN_BLOCK)) != JATTN_OK) return st;
  if ((st = make_map(&tk, k, BH, p.S, shape->d, 2, kv_rows)) != JATTN_OK) return st;
  if ((st = make_map(&tv, v, BH, p.S, shape->d, 2, kv_rows)) != JATTN_OK) return st;
  return jattn::launch_fwd_f16(p, shape->d, in_dtype == JATTN_BF16, tq, tk, tv,
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? JATTN_OK
             : JATTN_ERR_CUDA;
}

jattn_status jattn_fwd_fp8(const jattn_shape* shape, const void* q8, const void* k8, const void* v8,
                           const float* scales, void* o, float* lse, float softmax_scale, void* stream) {
  if (scales == nullptr || (reinterpret_cast<uintptr_t>(scales) & 3u)) return JATTN_ERR_INVALID_ARG;
  jattn::FwdParams p{};
  jattn_status st = fwd_common(shape, q8, k8, v8, o, lse, softmax_scale, p);
  if (st != JATTN_OK) return st;
  p.scales = scales;
  CUtensorMap tq, tk, tv;
  const int BH = p.B * p.H;
  const int kv_rows = jattn::fwd_kv_rows();
  if ((st = make_map(&tq, q8, BH, p.S, shape->d, 1, JATTN_BLOCK)) != JATTN_OK) return st;
  if ((st = make_map(&tk, k8, BH, p.S, shape->d, 1, kv_rows)) != JATTN_OK) return st;
  if ((st = make_map(&tv, v8, BH, p.S, shape->d, 1, kv_rows)) != JATTN_OK) return st;
  return jattn::launch_fwd_fp8(p, shape->d, tq, tk, tv, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? JATTN_OK
             : JATTN_ERR_CUDA;
}

// ---------------------------------------------------------------- high-precision 16-bit path

size_t jattn_rope_qkv_hp_workspace(const jattn_shape* shape) {
  if (check_shape(shape) != JATTN_OK) return 0;
  return hp_layout(shape).total;
}

jattn_status jattn_rope_qkv_hp(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                               const void* qkv_ref, const int32_t* pos, float theta, const int32_t split[3],
                               const float* norm_w, float eps, void* q, void* k, void* v, float* scales, void* qc,
                               void* kc, void* workspace, size_t workspace_bytes, void* stream) {
  jattn_status st = check_shape(shape);
  if (st != JATTN_OK) return st;
  if (norm_w != nullptr && (!(eps > 0.f) || !std::isfinite(eps))) return JATTN_ERR_INVALID_ARG;
  if (scales == nullptr || qc == nullptr || kc == nullptr || workspace == nullptr) return JATTN_ERR_INVALID_ARG;
  const HpLayout L = hp_layout(shape);
  if (workspace_bytes < L.total) return JATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return JATTN_ERR_ALIGNMENT;
  if (!aligned16(qc) || !aligned16(kc) || !aligned16(scales)) return JATTN_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* pair_stat = reinterpret_cast<float*>(ws + L.pair_stat);
  float* norm_r = reinterpret_cast<float*>(ws + L.norm_r);
  // 1. prologue: fp16 Q, K, V with power-of-two range scales, pair statistics
  st = rope_common(shape, qkv_txt, qkv_img, qkv_ref, pos, theta, split, norm_w, eps, JATTN_FP16, q, k, v, scales,
                   stream, nullptr, nullptr, pair_stat, norm_r);
  if (st != JATTN_OK) return st;
  // 2. pair selection and 3. correction rows
  jattn::CorrParams c{};
  const void* parts[3] = {qkv_txt, qkv_img, qkv_ref};
  const int lens[3] = {shape->S_txt, shape->S_img, shape->S_ref};
  for (int i = 0; i < 3; ++i) {
    c.src[i] = static_cast<const __nv_bfloat16*>(parts[i]);
    c.S_part[i] = lens[i];
    c.split[i] = split[i];
  }
  c.B = shape->B;
  c.H = shape->H;
  c.BH = shape->B * shape->H;
  c.S = total_S(shape);
  c.d = shape->d;
  c.nblk = n_blocks(c.S);
  c.pos = pos;
  c.theta = static_cast<double>(theta);
  c.rope = jattn::make_rope_table(c.theta, c.split, c.d);
  c.norm_w = norm_w;
  c.norm_r = norm_w != nullptr ? norm_r : nullptr;
  c.scales = scales;
  c.pair_stat = pair_stat;
  c.sel = reinterpret_cast<int32_t*>(ws + L.sel);
  c.qc = qc;
  c.kc = kc;
  return jattn::launch_qk_correction(c, static_cast<cudaStream_t>(stream)) == cudaSuccess ? JATTN_OK
                                                                                         : JATTN_ERR_CUDA;
}

jattn_status jattn_fwd_bf16_hp(const jattn_shape* shape, const void* q, const void* k, const void* v,
                               const float* scales, const void* qc, const void* kc, void* o, float* lse,
                               float softmax_scale, void* stream) {
  if (scales == nullptr || qc == nullptr || kc == nullptr) return JATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scales) & 3u) || !aligned16(qc) || !aligned16(kc)) return JATTN_ERR_ALIGNMENT;
  jattn::FwdParams p{};
  jattn_status st = fwd_common(shape, q, k, v, o, lse, softmax_scale, p);
  if (st != JATTN_OK) return st;
  p.scales = scales;
  CUtensorMap tq, tk, tv, tqc, tkc;
  const int BH = p.B * p.H;
  const int kv_rows = jattn::fwd_kv_rows();
  if ((st = make_map(&tq, q, BH, p.S, shape->d, 2, JATTN_BLOCK)) != JATTN_OK) return st;
  if ((st = make_map(&tk, k, BH, p.S, shape->d, 2, kv_rows)) != JATTN_OK) return st;
  if ((st = make_map(&tv, v, BH, p.S, shape->d, 2, kv_rows)) != JATTN_OK) return st;
  if ((st = make_map_corr(&tqc, qc, BH, p.S, JATTN_BLOCK)) != JATTN_OK) return st;
  if ((st = make_map_corr(&tkc, kc, BH, p.S, kv_rows)) != JATTN_OK) return st;
  return jattn::launch_fwd_f16_hp(p, shape->d, tq, tk, tv, tqc, tkc, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? JATTN_OK
             : JATTN_ERR_CUDA;
}

// ---------------------------------------------------------------- block-sparse attention

namespace {

struct SparseLayout {
  size_t pool, logits, list, count, total;
};

SparseLayout sparse_layout(const jattn_shape* shape) {
  const size_t BH = static_cast<size_t>(shape->B) * shape->H;
  const int S = total_S(shape);
  const size_t nb = n_blocks(S), nq = (S + 2 * JATTN_BLOCK - 1) / (2 * JATTN_BLOCK), d = shape->d;
  SparseLayout L{};
  size_t off = 0;
  auto seg = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
  L.pool = seg(2 * BH * nb * d * 4);
  L.logits = seg(BH * nq * nb * 4);
  L.list = seg(BH * nq * nb * 4);
  L.count = seg(BH * nq * 4);
  L.total = off;
  return L;
}

}  // namespace

size_t jattn_fwd_block_sparse_workspace(const jattn_shape* shape) {
  if (check_shape(shape) != JATTN_OK) return 0;
  return sparse_layout(shape).total;
}

jattn_status jattn_fwd_block_sparse(const jattn_shape* shape, jattn_dtype in_dtype, const void* q, const void* k,
                                    const void* v, float tau, void* workspace, size_t workspace_bytes, void* o,
                                    float* lse, int32_t* kv_list, int32_t* kv_count, float softmax_scale,
                                    void* stream) {
  if (in_dtype != JATTN_BF16 && in_dtype != JATTN_FP16) return JATTN_ERR_UNSUPPORTED;
  if (!(tau >= 0.f) || !std::isfinite(tau)) return JATTN_ERR_INVALID_ARG;
  jattn_status st = check_shape(shape);
  if (st != JATTN_OK) return st;
  const SparseLayout L = sparse_layout(shape);
  if (workspace == nullptr || workspace_bytes < L.total) return JATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return JATTN_ERR_ALIGNMENT;
  if ((kv_list != nullptr && (reinterpret_cast<uintptr_t>(kv_list) & 3u)) ||
      (kv_count != nullptr && (reinterpret_cast<uintptr_t>(kv_count) & 3u)))
    return JATTN_ERR_ALIGNMENT;
  jattn::FwdParams p{};
  if ((st = fwd_common(shape, q, k, v, o, lse, softmax_scale, p)) != JATTN_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  jattn::SparseParams sp{};
  sp.q = q;
  sp.k = k;
  sp.BH = p.B * p.H;
  sp.S = p.S;
  sp.d = shape->d;
  sp.nblk = p.n_kv;
  sp.n_qb = (p.n_tiles + 1) / 2;
  sp.scale = p.scale_log2 / 1.4426950408889634f;
  sp.tau = tau;
  sp.pool = reinterpret_cast<float*>(ws + L.pool);
  sp.logits = reinterpret_cast<float*>(ws + L.logits);
  sp.kv_list = kv_list != nullptr ? kv_list : reinterpret_cast<int32_t*>(ws + L.list);
  sp.kv_count = kv_count != nullptr ? kv_count : reinterpret_cast<int32_t*>(ws + L.count);
  if (jattn::launch_block_select(sp, in_dtype == JATTN_BF16, cs) != cudaSuccess) return JATTN_ERR_CUDA;
  p.kv_list = sp.kv_list;
  p.kv_count = sp.kv_count;
  CUtensorMap tq, tk, tv;
  const int BH = p.B * p.H;
  const int kv_rows = jattn::fwd_kv_rows();
  if ((st = make_map(&tq, q, BH, p.S, shape->d, 2, JATTN_BLOCK)) != JATTN_OK) return st;
  if ((st = make_map(&tk, k, BH, p.S, shape->d, 2, kv_rows)) != JATTN_OK) return st;
  if ((st = make_map(&tv, v, BH, p.S, shape->d, 2, kv_rows)) != JATTN_OK) return st;
  return jattn::launch_fwd_f16(p, shape->d, in_dtype == JATTN_BF16, tq, tk, tv, cs) == cudaSuccess ? JATTN_OK
                                                                                                  : JATTN_ERR_CUDA;
}

// ---------------------------------------------------------------- FP8 with token repair

int32_t jattn_repair_count(const jattn_shape* shape, float rho) {
  if (check_shape(shape) != JATTN_OK || !(rho >= 0.f && rho <= 1.f)) return -1;
  return repair_n(shape, rho);
}

size_t jattn_fwd_fp8_repair_workspace(const jattn_shape* shape, float rho) {
  if (check_shape(shape) != JATTN_OK || !(rho >= 0.f && rho <= 1.f)) return 0;
  return repair_layout(shape, repair_n(shape, rho)).total;
}

jattn_status jattn_fwd_fp8_repair(const jattn_shape* shape, const void* qkv_txt, const void* qkv_img,
                                  const void* qkv_ref, const int32_t* pos, float theta, const int32_t split[3],
                                  const float* norm_w, float eps, float rho, void* workspace,
                                  size_t workspace_bytes, void* o, float* lse, int32_t* repaired,
                                  float softmax_scale, void* stream) {
  jattn_status st = check_shape(shape);
  if (st != JATTN_OK) return st;
  if (!(rho >= 0.f && rho <= 1.f)) return JATTN_ERR_INVALID_ARG;
  if (norm_w != nullptr && (!(eps > 0.f) || !std::isfinite(eps))) return JATTN_ERR_INVALID_ARG;
  if (workspace == nullptr || o == nullptr) return JATTN_ERR_INVALID_ARG;
  const int n = repair_n(shape, rho);
  const RepairLayout L = repair_layout(shape, n);
  if (workspace_bytes < L.total) return JATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return JATTN_ERR_ALIGNMENT;
  if (repaired != nullptr && (reinterpret_cast<uintptr_t>(repaired) & 3u)) return JATTN_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int BH = shape->B * shape->H, S = total_S(shape), d = shape->d;
  float* scales = reinterpret_cast<float*>(ws + L.scales);
  float* score = reinterpret_cast<float*>(ws + L.score);
  int32_t* idx = repaired != nullptr ? repaired : reinterpret_cast<int32_t*>(ws + L.idx);
  uint32_t* kmask = reinterpret_cast<uint32_t*>(ws + L.kmask);
  float* lse_a = lse != nullptr ? lse : reinterpret_cast<float*>(ws + L.lse);

  // 1. Prologue: e4m3 Q/K/V + scales, and (with repairs) fp16 Q and the scores.
  st = rope_common(shape, qkv_txt, qkv_img, qkv_ref, pos, theta, split, norm_w, eps, JATTN_E4M3, ws + L.q8,
                   ws + L.k8, ws + L.v8, scales, stream, n > 0 ? ws + L.q16 : nullptr, n > 0 ? score : nullptr);
  if (st != JATTN_OK) return st;
  // 2. Selection and 3. exact keys / values of the selected tokens.
  if (n > 0) {
    if (jattn::launch_repair_select(score, BH, S, n, n_blocks(S), idx, kmask, cs) != cudaSuccess)
      return JATTN_ERR_CUDA;
    jattn::GatherParams g{};
    const void* parts[3] = {qkv_txt, qkv_img, qkv_ref};
    const int lens[3] = {shape->S_txt, shape->S_img, shape->S_ref};
    for (int i = 0; i < 3; ++i) {
      g.src[i] = static_cast<const __nv_bfloat16*>(parts[i]);
      g.S_part[i] = lens[i];
      g.split[i] = split[i];
    }
    g.B = shape->B;
    g.H = shape->H;
    g.S = S;
    g.d = d;
    g.n = n;
    g.pos = pos;
    g.theta = static_cast<double>(theta);
    g.rope = jattn::make_rope_table(g.theta, g.split, g.d);
    g.norm_w = norm_w;
    g.eps = eps;
    g.idx = idx;
    g.k_out = ws + L.kr;
    g.v_out = ws + L.vr;
    g.k8 = ws + L.k8;
    g.v8 = ws + L.v8;
    g.status = status_ptr();
    if (jattn::launch_repair_gather(g, cs) != cudaSuccess) return JATTN_ERR_CUDA;
  }
  // 4. 16-bit pass over the repaired keys: its partial O and LSE go to o and
  //    lse_a.  5. FP8 pass over the other keys, merged into them in its
  //    epilogue through the LSEs (the long pass has time to bring the partial
  //    rows into L2; the short one would wait on them).
  jattn::FwdParams p{};
  if ((st = fwd_common(shape, ws + L.q8, ws + L.k8, ws + L.v8, o, lse_a, softmax_scale, p)) != JATTN_OK) return st;
  CUtensorMap tq, tk, tv;
  const int kv_rows = jattn::fwd_kv_rows();
  if (n > 0) {
    jattn::FwdParams r = p;
    r.S_kv = n;
    r.n_kv = n_blocks(n);
    if ((st = make_map(&tq, ws + L.q16, BH, S, d, 2, JATTN_BLOCK)) != JATTN_OK) return st;
    if ((st = make_map(&tk, ws + L.kr, BH, n, d, 2, kv_rows)) != JATTN_OK) return st;
    if ((st = make_map(&tv, ws + L.vr, BH, n, d, 2, kv_rows)) != JATTN_OK) return st;
    if (jattn::launch_fwd_f16(r, d, false, tq, tk, tv, cs) != cudaSuccess) return JATTN_ERR_CUDA;
  }
  p.scales = scales;
  p.kmask = n > 0 ? kmask : nullptr;
  p.lse_prev = n > 0 ? lse_a : nullptr;
  p.lse = lse;
  if ((st = make_map(&tq, ws + L.q8, BH, S, d, 1, JATTN_BLOCK)) != JATTN_OK) return st;
  if ((st = make_map(&tk, ws + L.k8, BH, S, d, 1, kv_rows)) != JATTN_OK) return st;
  if ((st = make_map(&tv, ws + L.v8, BH, S, d, 1, kv_rows)) != JATTN_OK) return st;
  return jattn::launch_fwd_fp8(p, d, tq, tk, tv, cs) == cudaSuccess ? JATTN_OK : JATTN_ERR_CUDA;
}

jattn_status jattn_device_status(void* stream, int clear, uint32_t* bits) {
  uint32_t* ptr = status_ptr();
  if (ptr == nullptr) return JATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return JATTN_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpy(&w, ptr, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return JATTN_ERR_CUDA;
  if (clear && cudaMemset(ptr, 0, sizeof(uint32_t)) != cudaSuccess) return JATTN_ERR_CUDA;
  if (bits != nullptr) *bits = w;
  if (w & JATTN_DEV_CHECK) return JATTN_ERR_INTERNAL;
  if (w & JATTN_DEV_TIMEOUT) return JATTN_ERR_TIMEOUT;
  if (w & JATTN_DEV_RANGE) return JATTN_ERR_RANGE;
  return JATTN_OK;
}

jattn_status jattn_last_device_status(void* stream) { return jattn_device_status(stream, 0, nullptr); }

jattn_status jattn_selftest_wait_timeout(int32_t limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 10000) return JATTN_ERR_INVALID_ARG;
  uint32_t* ptr = status_ptr();
  if (ptr == nullptr) return JATTN_ERR_CUDA;
  return jattn::launch_selftest_wait(ptr, static_cast<uint64_t>(limit_ms) * 1000000ull,
                                     static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? JATTN_OK
             : JATTN_ERR_CUDA;
}

const char* jattn_status_string(jattn_status s) {
  switch (s) {
    case JATTN_OK: return "ok";
    case JATTN_ERR_INVALID_ARG: return "invalid argument";
    case JATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case JATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case JATTN_ERR_CUDA: return "CUDA error";
    case JATTN_ERR_TIMEOUT: return "device wait timed out";
    case JATTN_ERR_RANGE: return "value out of 16-bit range (saturated)";
    case JATTN_ERR_INTERNAL: return "kernel internal check failed";
  }
  return "unknown status";
}

const char* jattn_version(void) { return "0.1.0"; }

}  // extern "C"
