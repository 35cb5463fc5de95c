// The whole path on host buffers: copies in, prologue + attention, copy out,
// pipelined over (batch entry, head group) chunks so that the host<->device
// copies of one chunk overlap the kernels of another.  A head group is a
// strided slice of the [B, S, 3, H, d] inputs and of the [B, S, H, d]
// output, moved with 2-D copies into compact per-chunk device buffers, on
// which the device entry points run with H = heads per group.
//
// Three streams: the caller's stream runs the kernels; a copy-in and a
// copy-out stream (created once per thread and device, non-blocking) carry
// the transfers.  Ordering is by events only: the copy streams first wait
// for everything already enqueued on the caller's stream, batch entry b's
// kernels wait for its inputs, its output copy waits for its kernels, and
// the caller's stream finally waits for the last output copy -- so the call
// behaves as one operation on the caller's stream.  Events are re-recorded
// per batch entry (a wait binds to the record current when it is enqueued).
#include <cstdint>
#include <cuda_runtime.h>

#include "jattn.h"

namespace {

struct Pipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, ready = nullptr, done = nullptr, copied = nullptr;
  bool ok = false;
};

constexpr int kMaxDevices = 64;
thread_local Pipe t_pipe[kMaxDevices];

Pipe* pipe_for_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  Pipe& p = t_pipe[dev];
  if (!p.ok) {
    if (cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.ready, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.done, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.copied, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    p.ok = true;
  }
  return &p;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Heads per chunk: 2 (or 3) when that divides H, else all H.  Small chunks
// keep the pipeline's fill and drain short (the first chunk's copy-in and the
// last chunk's kernels and copy-out are not overlapped); at t2i_2048_base
// (H = 24) 12 groups per batch entry run within 1 ms of the copy-in alone.
int head_groups(int H) {
  for (int hg : {2, 3})
    if (H % hg == 0) return H / hg;
  return 1;
}

struct HostLayout {
  size_t part[3], pos, q, k, v, scales, scales_chunk, qc, kc, hp_ws, hp_ws_bytes, o, total;
};

bool valid_path(jattn_dtype path) { return path == JATTN_FP16 || path == JATTN_BF16 || path == JATTN_E4M3; }

// Every chunk (b, g) owns a compact slice of each buffer; the slices tile
// the buffers, so the sizes are those of the whole batch.
HostLayout host_layout(const jattn_shape* s, jattn_dtype path) {
  const size_t B = s->B, H = s->H, d = s->d, S = static_cast<size_t>(s->S_txt) + s->S_img + s->S_ref;
  const size_t lens[3] = {static_cast<size_t>(s->S_txt), static_cast<size_t>(s->S_img),
                          static_cast<size_t>(s->S_ref)};
  const size_t eb = path == JATTN_E4M3 ? 1 : 2;
  const size_t nb = (S + JATTN_BLOCK - 1) / JATTN_BLOCK;
  HostLayout L{};
  size_t off = 0;
  auto seg = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
  for (int i = 0; i < 3; ++i) L.part[i] = seg(B * lens[i] * 3 * H * d * 2);
  L.pos = seg(S * 3 * 4);
  L.q = seg(B * H * S * d * eb);
  L.k = seg(B * H * S * d * eb);
  L.v = seg(B * H * S * d * eb);
  // block scales (e4m3 scales, or the high-precision path's range scales),
  // one 256-byte aligned slice per chunk
  const size_t G = head_groups(s->H);
  L.scales_chunk = path == JATTN_BF16 ? 0 : align256(3 * (H / G) * nb * 4);
  L.scales = seg(B * G * L.scales_chunk);
  // the high-precision path (JATTN_FP16): correction rows, and one scratch
  // area of jattn_rope_qkv_hp that the chunks reuse in stream order
  const bool hp = path == JATTN_FP16;
  L.qc = seg(hp ? B * H * S * 16 * 2 : 0);
  L.kc = seg(hp ? B * H * S * 16 * 2 : 0);
  const jattn_shape one{1, static_cast<int>(H / G), s->S_txt, s->S_img, s->S_ref, s->d};
  L.hp_ws_bytes = hp ? jattn_rope_qkv_hp_workspace(&one) : 0;
  L.hp_ws = seg(L.hp_ws_bytes);
  L.o = seg(B * S * H * d * 2);
  L.total = off;
  return L;
}

bool shape_ok(const jattn_shape* s) {
  const int64_t S = s == nullptr ? 0 : static_cast<int64_t>(s->S_txt) + s->S_img + s->S_ref;
  return s != nullptr && s->B >= 1 && s->H >= 1 && s->H <= 65535 && s->S_txt >= 0 && s->S_img >= 0 &&
         s->S_ref >= 0 && (s->d == 64 || s->d == 128) && S >= 1 && S <= (1 << 24);
}

}  // namespace

extern "C" size_t jattn_joint_attention_host_workspace(const jattn_shape* shape, jattn_dtype path) {
  if (!shape_ok(shape) || !valid_path(path)) return 0;
  return host_layout(shape, path).total;
}

extern "C" jattn_status jattn_joint_attention_host(const jattn_shape* shape, const void* qkv_txt,
                                                   const void* qkv_img, const void* qkv_ref, const int32_t* pos,
                                                   float theta, const int32_t split[3], jattn_dtype path, void* o,
                                                   float softmax_scale, void* workspace, size_t workspace_bytes,
                                                   void* stream) {
  if (shape == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!valid_path(path)) return JATTN_ERR_UNSUPPORTED;
  if (!shape_ok(shape)) {
    // the device entry points report which argument is wrong
    return shape->d != 64 && shape->d != 128 ? JATTN_ERR_UNSUPPORTED : JATTN_ERR_INVALID_ARG;
  }
  const void* parts[3] = {qkv_txt, qkv_img, qkv_ref};
  const int lens[3] = {shape->S_txt, shape->S_img, shape->S_ref};
  for (int i = 0; i < 3; ++i)
    if (lens[i] > 0 && parts[i] == nullptr) return JATTN_ERR_INVALID_ARG;
  if (pos == nullptr || o == nullptr || split == nullptr || workspace == nullptr) return JATTN_ERR_INVALID_ARG;
  // The per-entry device calls check these too; checking them here keeps an
  // argument error from surfacing after copies were already enqueued.
  if (!(theta > 0.f) || theta == INFINITY) return JATTN_ERR_INVALID_ARG;
  if (split[0] < 0 || split[1] < 0 || split[2] < 0 || ((split[0] | split[1] | split[2]) & 1) ||
      split[0] + split[1] + split[2] != shape->d)
    return JATTN_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || softmax_scale == INFINITY || softmax_scale == -INFINITY)
    return JATTN_ERR_INVALID_ARG;
  const HostLayout L = host_layout(shape, path);
  if (workspace_bytes < L.total) return JATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return JATTN_ERR_ALIGNMENT;

  Pipe* P = pipe_for_device();
  if (P == nullptr) return JATTN_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int B = shape->B, H = shape->H, d = shape->d;
  const int G = head_groups(H), Hg = H / G;
  const int S = shape->S_txt + shape->S_img + shape->S_ref;
  const size_t eb = path == JATTN_E4M3 ? 1 : 2;
  const size_t row_in = static_cast<size_t>(H) * d * 2;          // host input: one (token, Q|K|V) row
  const size_t row_grp = static_cast<size_t>(Hg) * d * 2;        // the group's part of it
  const size_t lay_c = static_cast<size_t>(Hg) * S * d * eb;     // one chunk of laid-out q / k / v
  const size_t out_c = static_cast<size_t>(S) * Hg * d * 2;      // one chunk of o
  const jattn_shape one{1, Hg, shape->S_txt, shape->S_img, shape->S_ref, d};

#define JATTN_CU(x) do { if ((x) != cudaSuccess) return JATTN_ERR_CUDA; } while (0)
  JATTN_CU(cudaEventRecord(P->start, cs));
  JATTN_CU(cudaStreamWaitEvent(P->in, P->start, 0));
  JATTN_CU(cudaStreamWaitEvent(P->out, P->start, 0));
  JATTN_CU(cudaMemcpyAsync(ws + L.pos, pos, static_cast<size_t>(S) * 3 * 4, cudaMemcpyHostToDevice, P->in));
  for (int b = 0; b < B; ++b) {
    for (int g = 0; g < G; ++g) {
      const size_t c = static_cast<size_t>(b) * G + g;           // chunk index
      const void* dparts[3] = {nullptr, nullptr, nullptr};
      for (int i = 0; i < 3; ++i) {
        if (lens[i] == 0) continue;
        const size_t rows = static_cast<size_t>(lens[i]) * 3;     // (token, Q|K|V) rows of this stream
        uint8_t* dst = ws + L.part[i] + c * rows * row_grp;
        const uint8_t* src = static_cast<const uint8_t*>(parts[i]) + b * rows * row_in + g * row_grp;
        JATTN_CU(cudaMemcpy2DAsync(dst, row_grp, src, row_in, row_grp, rows, cudaMemcpyHostToDevice, P->in));
        dparts[i] = dst;
      }
      JATTN_CU(cudaEventRecord(P->ready, P->in));
      JATTN_CU(cudaStreamWaitEvent(cs, P->ready, 0));
      void* q = ws + L.q + c * lay_c;
      void* k = ws + L.k + c * lay_c;
      void* v = ws + L.v + c * lay_c;
      void* oc = ws + L.o + c * out_c;
      const int32_t* dpos = reinterpret_cast<const int32_t*>(ws + L.pos);
      jattn_status st;
      if (path == JATTN_E4M3) {
        float* sc = reinterpret_cast<float*>(ws + L.scales + c * L.scales_chunk);
        st = jattn_rope_qkv(&one, dparts[0], dparts[1], dparts[2], dpos, theta, split, JATTN_E4M3, q, k, v, sc, cs);
        if (st == JATTN_OK) st = jattn_fwd_fp8(&one, q, k, v, sc, oc, nullptr, softmax_scale, cs);
      } else if (path == JATTN_FP16) {
        // the high-precision 16-bit pair
        float* sc = reinterpret_cast<float*>(ws + L.scales + c * L.scales_chunk);
        void* qc = ws + L.qc + c * static_cast<size_t>(Hg) * S * 32;
        void* kc = ws + L.kc + c * static_cast<size_t>(Hg) * S * 32;
        st = jattn_rope_qkv_hp(&one, dparts[0], dparts[1], dparts[2], dpos, theta, split, nullptr, 0.f, q, k, v, sc,
                               qc, kc, ws + L.hp_ws, L.hp_ws_bytes, cs);
        if (st == JATTN_OK) st = jattn_fwd_bf16_hp(&one, q, k, v, sc, qc, kc, oc, nullptr, softmax_scale, cs);
      } else {
        st = jattn_rope_qkv(&one, dparts[0], dparts[1], dparts[2], dpos, theta, split, path, q, k, v, nullptr, cs);
        if (st == JATTN_OK) st = jattn_fwd_bf16(&one, path, q, k, v, oc, nullptr, softmax_scale, cs);
      }
      if (st != JATTN_OK) return st;
      JATTN_CU(cudaEventRecord(P->done, cs));
      JATTN_CU(cudaStreamWaitEvent(P->out, P->done, 0));
      // o chunk [S][Hg][d] -> host o[b][s][g*Hg .. g*Hg+Hg)[d]
      uint8_t* dst = static_cast<uint8_t*>(o) + static_cast<size_t>(b) * S * row_in + g * row_grp;
      JATTN_CU(cudaMemcpy2DAsync(dst, row_in, oc, row_grp, row_grp, S, cudaMemcpyDeviceToHost, P->out));
    }
  }
  JATTN_CU(cudaEventRecord(P->copied, P->out));
  JATTN_CU(cudaStreamWaitEvent(cs, P->copied, 0));
  // A later call starts by waiting on the caller's stream, which now
  // includes everything above, so its copies cannot overrun this call's
  // kernels.
#undef JATTN_CU
  return JATTN_OK;
}
