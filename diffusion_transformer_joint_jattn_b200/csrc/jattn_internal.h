// Parameter blocks and launchers shared by the C-ABI layer (jattn_api.cu)
// and the kernel translation units.  Not part of the public interface.
#pragma once

#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace jattn {

// Rotary frequencies of the d/2 channel pairs, built on the host once per
// call: pair p lies on axis axis[p] (0 = t, 1 = row, 2 = col: spans of
// split[0], split[1], split[2] channels in that order) and turns by
// pos_axis * omega[p], omega[p] = theta^(-2i/n) for its index i inside its
// axis span of n channels.  Passed by value in the kernel parameters.
struct RopeTable {
  double omega[64];
  uint8_t axis[64];
};

inline RopeTable make_rope_table(double theta, const int split[3], int d) {
  RopeTable t{};
  for (int p = 0; p < d / 2 && p < 64; ++p) {
    int axis, i, n;
    if (p < split[0] / 2) { axis = 0; i = p; n = split[0]; }
    else if (p < (split[0] + split[1]) / 2) { axis = 1; i = p - split[0] / 2; n = split[1]; }
    else { axis = 2; i = p - (split[0] + split[1]) / 2; n = split[2]; }
    t.axis[p] = static_cast<uint8_t>(axis);
    t.omega[p] = std::pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(n));
  }
  return t;
}

struct RopeParams {
  const __nv_bfloat16* src[3];  // txt, img, ref streams [B, S_part, 3, H, d]
  int S_part[3];
  int B, H, S, d, nblk;
  const int32_t* pos;           // [S, 3]
  double theta;
  int split[3];
  RopeTable rope;               // frequencies of theta / split (make_rope_table)
  void* dst[3];                 // q, k, v [B, H, S, d]
  float* scales;                // e4m3 output: [3][B][H][nblk]
  const float* norm_w;          // query/key RMSNorm weights [3][2][d], or null
  float eps;                    // RMSNorm epsilon
  void* q16;                    // e4m3 output with token repair: also fp16 Q [B, H, S, d], else null
  float* score;                 // with token repair: [2][B, H, S], |k|^2 then |v|^2 per token, else null
  int hp;                       // fp16 output of the high-precision path: power-of-two range scales in
                                //   `scales` ([3][B][H][nblk]), pair statistics and norm factors below
  float* pair_stat;             // hp: [2][B*H][nblk][d/2] max squared channel-pair norm over each block
  float* norm_r;                // hp with norm_w: [2][B*H][S] RMSNorm factor of every Q / K row
  uint32_t* status;
};

// Exact (16-bit) keys and values of the repaired tokens.
struct GatherParams {
  const __nv_bfloat16* src[3];  // txt, img, ref streams [B, S_part, 3, H, d]
  int S_part[3];
  int B, H, S, d, n;            // n repaired tokens per (b, h)
  const int32_t* pos;           // [S, 3]
  double theta;
  int split[3];
  RopeTable rope;
  const float* norm_w;          // as RopeParams
  float eps;
  const int32_t* idx;           // [B*H][n] token indices
  void* k_out;                  // fp16 [B*H][n][d], rotated (and normalised) keys
  void* v_out;                  // fp16 [B*H][n][d]
  uint8_t* k8;                  // e4m3 [B*H][S][d] keys / values of the FP8 pass: the repaired
  uint8_t* v8;                  //   tokens' rows are set to code 0 (logit exactly 0, value 0)
  uint32_t* status;
};

cudaError_t launch_repair_gather(const GatherParams& p, cudaStream_t st);
// Per (b, h): the n largest scores |k|^2 + |v|^2 (ties to the lower index)
// -> idx [B*H][n] in index order, and the key mask [B*H][n_kv][4] words with
// their bits set.  score holds the [2][B*H][S] K and V planes; the K plane is
// overwritten with the sums.
cudaError_t launch_repair_select(float* score, int BH, int S, int n, int n_kv, int32_t* idx,
                                 uint32_t* kmask, cudaStream_t st);

// High-precision 16-bit path: channel pairs per (b, h) whose rotated Q / K
// values get an fp16 low part, and the columns of one correction row
// (hi and lo of 2 * kCorrPairs channels).
constexpr int kCorrPairs = 4;
constexpr int kCorrCols = 4 * kCorrPairs;

struct CorrParams {
  const __nv_bfloat16* src[3];  // txt, img, ref streams [B, S_part, 3, H, d]
  int S_part[3];
  int B, H, BH, S, d, nblk;
  const int32_t* pos;           // [S, 3]
  double theta;
  int split[3];
  RopeTable rope;
  const float* norm_w;          // query/key RMSNorm weights [3][2][d], or null
  const float* norm_r;          // with norm_w: [2][B*H][S] row factors written by the prologue
  const float* scales;          // [3][B][H][nblk] power-of-two range scales written by the prologue
  const float* pair_stat;       // [2][B*H][nblk][d/2] written by the prologue
  int32_t* sel;                 // [B*H][kCorrPairs] selected pairs, ascending
  void* qc;                     // fp16 [B*H][S][kCorrCols]: [hi | lo] of the selected Q channels
  void* kc;                     // fp16 [B*H][S][kCorrCols]: [lo | hi] of the selected K channels
};

cudaError_t launch_qk_correction(const CorrParams& p, cudaStream_t st);

// Block-sparse attention: selection of the key tiles each 256-row query
// block attends to.
struct SparseParams {
  const void* q;                // [B*H][S][d] 16-bit (rotated)
  const void* k;
  int BH, S, d, nblk, n_qb;     // nblk = ceil(S / 128) key tiles, n_qb = ceil(S / 256) query blocks
  float scale;                  // softmax scale
  float tau;                    // keep a key block iff its estimated share >= tau / nblk
  float* pool;                  // [2][B*H][nblk][d] column sums of every 128-token tile of Q, K
  float* logits;                // [B*H][n_qb][nblk] block logits (scratch of the selection)
  int32_t* kv_list;             // [B*H][n_qb][nblk] kept key tiles, ascending (first kv_count entries)
  int32_t* kv_count;            // [B*H][n_qb]
};

cudaError_t launch_block_select(const SparseParams& p, bool in_bf16, cudaStream_t st);

struct QuantParams {
  const void* x;                // [BH, S, d] 16-bit
  void* x8;                     // [BH, S, d] e4m3
  float* scales;                // [BH][nblk]
  int BH, S, d, nblk;
};

struct FwdParams {
  int B, H, S, n_tiles;         // queries: S rows, n_tiles = ceil(S / 128)
  int S_kv, n_kv;               // keys: S_kv rows (= S except for a residual pass), n_kv = ceil(S_kv / 128)
  float scale_log2;             // softmax_scale * log2(e)
  __nv_bfloat16* o;             // [B, S, H, d]
  float* lse;                   // [B, H, S] or null
  const float* scales;          // fp8 and the high-precision fp16 path: [3][B][H][n_tiles]
  const uint32_t* kmask;        // null, or [B*H][n_kv][4] words: bit set = key left out of this pass
  const float* lse_prev;        // null, or [B, H, S]: o already holds a partial result with this
                                // LSE over other keys; the pass merges its own into o (and lse)
  const int32_t* kv_list;       // null, or [B*H][n_qp][n_kv]: the key tiles each pair of query
  const int32_t* kv_count;      //   tiles walks, ascending, and how many ([B*H][n_qp]); n_qp =
                                //   ceil(n_tiles / 2); every count >= 1
  uint32_t* status;
  uint64_t timeout_ns;
  long long* trace;             // development timing probe; always null in the library
};

// out_kind: 0 = fp16, 1 = bf16, 2 = e4m3
cudaError_t launch_rope_qkv(const RopeParams& p, int out_kind, cudaStream_t st);
cudaError_t launch_quant_fp8(const QuantParams& p, bool in_bf16, cudaStream_t st);

// 16-bit forward (in_bf16 selects the operand type) and e4m3 forward.  The
// tensor maps describe q, k, v as 3-D [BH][S][d] with 128-row boxes.
cudaError_t launch_fwd_f16(const FwdParams& p, int d, bool in_bf16, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st);
cudaError_t launch_fwd_fp8(const FwdParams& p, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, cudaStream_t st);
// High-precision 16-bit forward: fp16 operands with power-of-two block scales
// in p.scales and the correction tiles described by tqc / tkc ([BH][S][16]
// fp16, 32-byte swizzle, 128-row boxes).
cudaError_t launch_fwd_f16_hp(const FwdParams& p, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const CUtensorMap& tqc, const CUtensorMap& tkc,
                              cudaStream_t st);

// Rows of the K / V tiles the forward kernels walk (the TMA box height).
int fwd_kv_rows();

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t st);

// Unique id of the calling thread's current CUDA context (0 when there is
// none or it cannot be read).  Device addresses of file-scope __device__
// variables are cached per context: a cudaDeviceReset makes a new context,
// whose id differs, and the address is looked up again.
unsigned long long current_context_id();

}  // namespace jattn
