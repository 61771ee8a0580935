// attn_api.cu -- the extern "C" entry points declared in include/attn_b200.h:
// argument validation, the per-device error word, and dispatch to the
// kernel launchers.  No device memory is allocated here or anywhere in the
// library.
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>
#include <pthread.h>

#include "attn_b200.h"
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace attn {

// One error word per device that has loaded the library.
__device__ unsigned int g_error_word = 0;

unsigned int* device_error_word() {
  constexpr int kMaxDevices = 64;
  static unsigned int* addr[kMaxDevices] = {};
  static pthread_mutex_t mu = PTHREAD_MUTEX_INITIALIZER;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  pthread_mutex_lock(&mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess) addr[dev] = static_cast<unsigned int*>(p);
  }
  unsigned int* a = addr[dev];
  pthread_mutex_unlock(&mu);
  return a;
}

}  // namespace attn

namespace attn {
namespace {
__global__ void fill_neg_inf_kernel(float* p, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = -INFINITY;
}
}  // namespace

cudaError_t fill_neg_inf(float* p, size_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const size_t want = (n + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(want < 4096 ? want : 4096);
  fill_neg_inf_kernel<<<blocks, 256, 0, stream>>>(p, n);
  return cudaGetLastError();
}
}  // namespace attn

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

attn_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA; }

attn_status_t check_prefill(const void* q, const void* k, const void* v, const void* out, int B, int Hq, int Hkv,
                            int Sq, int Skv, int D, float scale, int causal, int window) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Sq < 0 || Skv < 0 || D <= 0 || window < 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0 || Sq == 0) return ATTN_OK;  // nothing to do (checked again by the caller)
  if (Hkv == 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  // with no keys (Skv == 0) k and v are never read and may be null
  if (q == nullptr || out == nullptr || (Skv > 0 && (k == nullptr || v == nullptr))) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_INVALID_ARG;
  if (window > 0 && !causal) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq > 65535LL * 32768LL) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

}  // namespace

extern "C" {

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_BAD_PAGE: return "ATTN_ERR_BAD_PAGE";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    case ATTN_ERR_OUT_OF_PAGES: return "ATTN_ERR_OUT_OF_PAGES";
  }
  return "ATTN_ERR_UNKNOWN";
}

int attn_version(void) { return 103; }

}  // extern "C"

namespace {

attn_status_t prefill_bf16(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                           int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
                           attn_stream_t stream) {
  const attn_status_t st = check_prefill(q, k, v, out, B, Hq, Hkv, Sq, Skv, D, scale, causal, window);
  if (st != ATTN_OK || B == 0 || Hq == 0 || Sq == 0) return st;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (Skv == 0) {  // no key at all: every row is empty, its output 0 and its lse -inf
    if (cudaMemsetAsync(out, 0, static_cast<size_t>(B) * Hq * Sq * D * 2, s) != cudaSuccess) return ATTN_ERR_CUDA;
    return lse == nullptr ? ATTN_OK : from_cuda(attn::fill_neg_inf(lse, static_cast<size_t>(B) * Hq * Sq, s));
  }
  return from_cuda(attn::launch_prefill_tc(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, window,
                                           attn::device_error_word(), s));
}

attn_status_t prefill_f32(const float* q, const float* k, const float* v, float* out, float* lse, int B, int Hq,
                          int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
                          attn_stream_t stream) {
  const attn_status_t st = check_prefill(q, k, v, out, B, Hq, Hkv, Sq, Skv, D, scale, causal, window);
  if (st != ATTN_OK || B == 0 || Hq == 0 || Sq == 0) return st;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * Hq > 65535) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (Skv == 0) {
    if (cudaMemsetAsync(out, 0, static_cast<size_t>(B) * Hq * Sq * D * sizeof(float), s) != cudaSuccess)
      return ATTN_ERR_CUDA;
    return lse == nullptr ? ATTN_OK : from_cuda(attn::fill_neg_inf(lse, static_cast<size_t>(B) * Hq * Sq, s));
  }
  return from_cuda(attn::launch_prefill_f32(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, s));
}

}  // namespace

extern "C" {

attn_status_t attn_prefill(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv, int Sq,
                           int Skv, int D, float scale, int causal, int window, attn_stream_t stream) {
  return prefill_bf16(q, k, v, out, nullptr, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, stream);
}

attn_status_t attn_prefill_lse(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                               int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
                               attn_stream_t stream) {
  if (lse == nullptr && B > 0 && Hq > 0 && Sq > 0) return ATTN_ERR_INVALID_ARG;
  return prefill_bf16(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, stream);
}

attn_status_t attn_prefill_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                 const int32_t* seq_lens, int page_size, int B, int Hq, int Hkv, int Sq, int D,
                                 int num_pages, int max_pages, int max_seq_len, float scale, int causal, int window,
                                 void* out, float* lse, attn_stream_t stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Sq < 0 || D <= 0 || num_pages < 0 || max_pages < 0 || max_seq_len < 0 ||
      window < 0 || page_size <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0 || Sq == 0) return ATTN_OK;
  if (Hkv == 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (q == nullptr || out == nullptr || seq_lens == nullptr) return ATTN_ERR_INVALID_ARG;
  if (max_seq_len > 0 && (k_pool == nullptr || v_pool == nullptr || page_table == nullptr || max_pages == 0 ||
                          num_pages == 0))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_INVALID_ARG;
  if (window > 0 && !causal) return ATTN_ERR_UNSUPPORTED;
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128 && page_size != 256)
    return ATTN_ERR_UNSUPPORTED;
  // TMA plane coordinates (page * Hkv + g, one page past the pool for boxes past a sequence end) are int32
  if ((static_cast<long long>(num_pages) + 1) * Hkv > 0x7FFFFFFFLL) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (max_seq_len == 0) {  // every cache is empty: outputs 0, lse -inf
    if (cudaMemsetAsync(out, 0, static_cast<size_t>(B) * Hq * Sq * D * 2, s) != cudaSuccess) return ATTN_ERR_CUDA;
    return lse == nullptr ? ATTN_OK : from_cuda(attn::fill_neg_inf(lse, static_cast<size_t>(B) * Hq * Sq, s));
  }
  return from_cuda(attn::launch_prefill_tc_paged(q, k_pool, v_pool, page_table, seq_lens, page_size, B, Hq, Hkv, Sq,
                                                 D, num_pages, max_pages, max_seq_len, scale, causal, window, out, lse,
                                                 attn::device_error_word(), s));
}

// attn_prefill from and to host memory.  The work is cut into pieces of
// consecutive (batch, kv head) pairs, each with its query heads: a piece is
// contiguous in q, k, v and out, so each of its transfers is one copy, and
// its kernel is an attn_prefill over one batch element of Hkv' = pairs kv
// heads.  Piece i's input copy (copy_in) overlaps piece i-1's kernel
// (stream) and piece i-2's output copy (copy_out).
attn_status_t attn_prefill_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                                void* q_dev, void* k_dev, void* v_dev, void* out_dev, int B, int Hq, int Hkv,
                                int Sq, int Skv, int D, float scale, int causal, int window, int chunks,
                                attn_stream_t stream, attn_stream_t copy_in, attn_stream_t copy_out) {
  attn_status_t st = check_prefill(q_dev, k_dev, v_dev, out_dev, B, Hq, Hkv, Sq, Skv, D, scale, causal, window);
  if (st != ATTN_OK || B == 0 || Hq == 0 || Sq == 0) return st;
  if (q_host == nullptr || out_host == nullptr || (Skv > 0 && (k_host == nullptr || v_host == nullptr)))
    return ATTN_ERR_INVALID_ARG;
  const long long units = static_cast<long long>(B) * Hkv;   // (batch, kv head) pairs
  const int G = Hq / Hkv;
  const size_t q_unit = static_cast<size_t>(G) * Sq * D * 2;   // bytes of q (and out) per pair
  const size_t kv_unit = static_cast<size_t>(Skv) * D * 2;     // bytes of k (and v) per pair
  if (chunks < 0 || chunks > units) return ATTN_ERR_INVALID_ARG;
  // The host link bounds this call, not the kernels.  The last piece's kernel
  // and copy back follow the last input copy, so more pieces shorten the
  // tail, while every piece adds some tens of microseconds of copy and launch
  // latency.  Measured on B200 (PCIe, pinned buffers): a 38 MB input did best
  // in 2 pieces; 201 MB inputs in 4 to 8 (5.6 ms in 2 pieces, 5.0 in 4, a
  // little over or under that in 8).  Default: one piece per 48 MB of input,
  // rounded, between 2 and 8.
  if (chunks == 0) {
    const long long in_mb = static_cast<long long>((units * (q_unit + 2 * kv_unit)) >> 20);
    long long c = (in_mb + 24) / 48;
    c = c < 2 ? 2 : (c > 8 ? 8 : c);
    chunks = static_cast<int>(c < units ? c : units);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t si = copy_in != nullptr ? reinterpret_cast<cudaStream_t>(copy_in) : s;
  cudaStream_t so = copy_out != nullptr ? reinterpret_cast<cudaStream_t>(copy_out) : s;
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};   // entry / inputs of a piece on the device / its output ready
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) st = ATTN_ERR_CUDA;
  // the copies wait for earlier work on `stream` (which may still use the device buffers)
  if (st == ATTN_OK && (cudaEventRecord(ev[0], s) != cudaSuccess || cudaStreamWaitEvent(si, ev[0], 0) != cudaSuccess ||
                        cudaStreamWaitEvent(so, ev[0], 0) != cudaSuccess))
    st = ATTN_ERR_CUDA;
  const char* qh = static_cast<const char*>(q_host);
  const char* kh = static_cast<const char*>(k_host);
  const char* vh = static_cast<const char*>(v_host);
  char* oh = static_cast<char*>(out_host);
  char* qd = static_cast<char*>(q_dev);
  char* kd = static_cast<char*>(k_dev);
  char* vd = static_cast<char*>(v_dev);
  char* od = static_cast<char*>(out_dev);
  for (int c = 0; c < chunks && st == ATTN_OK; ++c) {
    const long long u0 = units * c / chunks, u1 = units * (c + 1) / chunks;
    if (u1 <= u0) continue;
    const size_t n = static_cast<size_t>(u1 - u0);
    const size_t qo = static_cast<size_t>(u0) * q_unit, ko = static_cast<size_t>(u0) * kv_unit;
    if (cudaMemcpyAsync(qd + qo, qh + qo, n * q_unit, cudaMemcpyHostToDevice, si) != cudaSuccess ||
        (kv_unit > 0 && (cudaMemcpyAsync(kd + ko, kh + ko, n * kv_unit, cudaMemcpyHostToDevice, si) != cudaSuccess ||
                         cudaMemcpyAsync(vd + ko, vh + ko, n * kv_unit, cudaMemcpyHostToDevice, si) != cudaSuccess)) ||
        cudaEventRecord(ev[1], si) != cudaSuccess || cudaStreamWaitEvent(s, ev[1], 0) != cudaSuccess) {
      st = ATTN_ERR_CUDA;
      break;
    }
    st = prefill_bf16(qd + qo, kv_unit > 0 ? kd + ko : nullptr, kv_unit > 0 ? vd + ko : nullptr, od + qo, nullptr, 1,
                      static_cast<int>(n) * G, static_cast<int>(n), Sq, Skv, D, scale, causal, window, stream);
    if (st != ATTN_OK) break;
    if (cudaEventRecord(ev[2], s) != cudaSuccess || cudaStreamWaitEvent(so, ev[2], 0) != cudaSuccess ||
        cudaMemcpyAsync(oh + qo, od + qo, n * q_unit, cudaMemcpyDeviceToHost, so) != cudaSuccess)
      st = ATTN_ERR_CUDA;
  }
  // later work on `stream` comes after every copy this call enqueued, also
  // when a piece failed part way
  if (ev[1] != nullptr && ev[2] != nullptr) {
    const bool joined = cudaEventRecord(ev[1], si) == cudaSuccess && cudaStreamWaitEvent(s, ev[1], 0) == cudaSuccess &&
                        cudaEventRecord(ev[2], so) == cudaSuccess && cudaStreamWaitEvent(s, ev[2], 0) == cudaSuccess;
    if (!joined && st == ATTN_OK) st = ATTN_ERR_CUDA;
  }
  for (auto& e : ev)
    if (e != nullptr) cudaEventDestroy(e);   // released once the recorded work completes
  return st;
}

attn_status_t attn_prefill_f32(const float* q, const float* k, const float* v, float* out, int B, int Hq, int Hkv,
                               int Sq, int Skv, int D, float scale, int causal, int window, attn_stream_t stream) {
  return prefill_f32(q, k, v, out, nullptr, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, stream);
}

attn_status_t attn_prefill_f32_lse(const float* q, const float* k, const float* v, float* out, float* lse, int B,
                                   int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
                                   attn_stream_t stream) {
  if (lse == nullptr && B > 0 && Hq > 0 && Sq > 0) return ATTN_ERR_INVALID_ARG;
  return prefill_f32(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, stream);
}

size_t attn_decode_paged_workspace_size(int N, int Hq, int D, int max_seq_len, int page_size) {
  if (N < 0 || Hq < 0 || D <= 0 || max_seq_len < 0 || page_size <= 0) return 0;
  return attn::decode_workspace_bytes(N, Hq, D, max_seq_len, page_size);
}

}  // extern "C"

namespace {

// Argument checks of the paged decode; ATTN_OK also for an empty batch (N or Hq 0).
attn_status_t decode_paged_check(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                 const int32_t* seq_lens, int page_size, int N, int Hq, int Hkv, int D, int num_pages,
                                 int max_pages, int max_seq_len, float scale, int window, const void* workspace,
                                 size_t workspace_bytes, const void* out, float k_scale, float v_scale) {
  if (N < 0 || Hq < 0 || Hkv < 0 || D <= 0 || num_pages < 0 || max_pages < 0 || max_seq_len < 0 || window < 0 ||
      page_size <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale))
    return ATTN_ERR_INVALID_ARG;
  if (N == 0 || Hq == 0) return ATTN_OK;
  if (Hkv == 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (q == nullptr || out == nullptr || seq_lens == nullptr) return ATTN_ERR_INVALID_ARG;
  if (max_seq_len > 0 && (k_pool == nullptr || v_pool == nullptr || page_table == nullptr || max_pages == 0))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return ATTN_ERR_UNSUPPORTED;
  if (page_size % 16 != 0 || page_size > 256) return ATTN_ERR_UNSUPPORTED;
  if (N > 65535 || Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
  const size_t need = attn::decode_workspace_bytes(N, Hq, D, max_seq_len, page_size);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return ATTN_ERR_WORKSPACE;
  return ATTN_OK;
}

attn_status_t decode_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                           const int32_t* seq_lens, int page_size, int N, int Hq, int Hkv, int D, int num_pages,
                           int max_pages, int max_seq_len, float scale, int window, void* workspace,
                           size_t workspace_bytes, void* out, attn_stream_t stream, bool fp8, float k_scale,
                           float v_scale) {
  const attn_status_t st = decode_paged_check(q, k_pool, v_pool, page_table, seq_lens, page_size, N, Hq, Hkv, D,
                                              num_pages, max_pages, max_seq_len, scale, window, workspace,
                                              workspace_bytes, out, k_scale, v_scale);
  if (st != ATTN_OK || N == 0 || Hq == 0) return st;
  return from_cuda(attn::launch_decode_paged(q, k_pool, v_pool, page_table, seq_lens, page_size, N, Hq, Hkv, D,
                                             num_pages, max_pages, max_seq_len, scale, window, workspace, out,
                                             attn::device_error_word(), reinterpret_cast<cudaStream_t>(stream), fp8,
                                             k_scale, v_scale));
}

}  // namespace

extern "C" {

attn_status_t attn_decode_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                const int32_t* seq_lens, int page_size, int N, int Hq, int Hkv, int D,
                                int num_pages, int max_pages, int max_seq_len, float scale, int window,
                                void* workspace, size_t workspace_bytes, void* out, attn_stream_t stream) {
  return decode_paged(q, k_pool, v_pool, page_table, seq_lens, page_size, N, Hq, Hkv, D, num_pages, max_pages,
                      max_seq_len, scale, window, workspace, workspace_bytes, out, stream, false, 1.f, 1.f);
}

attn_status_t attn_decode_paged_fp8(const void* q, const uint8_t* k_pool, const uint8_t* v_pool,
                                    const int32_t* page_table, const int32_t* seq_lens, int page_size, int N, int Hq,
                                    int Hkv, int D, int num_pages, int max_pages, int max_seq_len, float scale,
                                    float k_scale, float v_scale, int window, void* workspace,
                                    size_t workspace_bytes, void* out, attn_stream_t stream) {
  return decode_paged(q, k_pool, v_pool, page_table, seq_lens, page_size, N, Hq, Hkv, D, num_pages, max_pages,
                      max_seq_len, scale, window, workspace, workspace_bytes, out, stream, true, k_scale, v_scale);
}

// One serving decode step from and to host memory: copy the step's inputs in,
// append the new token's K/V, decode, copy the output out, in that order on
// `stream` (every check happens before anything is enqueued).
attn_status_t attn_decode_step_host(const void* q_host, const void* k_new_host, const void* v_new_host,
                                    void* out_host, void* q_dev, void* k_new_dev, void* v_new_dev, void* out_dev,
                                    void* k_pool, void* v_pool, const int32_t* page_table, const int32_t* seq_lens,
                                    int page_size, int N, int Hq, int Hkv, int D, int num_pages, int max_pages,
                                    int max_seq_len, float scale, int window, void* workspace,
                                    size_t workspace_bytes, attn_stream_t stream) {
  if (N < 0 || Hq < 0 || Hkv < 0 || D <= 0) return ATTN_ERR_INVALID_ARG;
  if (N == 0 || Hq == 0) return ATTN_OK;
  if (q_host == nullptr || k_new_host == nullptr || v_new_host == nullptr || out_host == nullptr ||
      q_dev == nullptr || k_new_dev == nullptr || v_new_dev == nullptr || out_dev == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k_new_dev) || !aligned16(v_new_dev)) return ATTN_ERR_INVALID_ARG;
  // the decode's own checks (the append's are a subset for S_new = 1), before any copy is enqueued
  attn_status_t st = decode_paged_check(q_dev, k_pool, v_pool, page_table, seq_lens, page_size, N, Hq, Hkv, D,
                                        num_pages, max_pages, max_seq_len, scale, window, workspace,
                                        workspace_bytes, out_dev, 1.f, 1.f);
  if (st != ATTN_OK) return st;
  if (max_seq_len == 0 || max_pages == 0 || num_pages == 0) return ATTN_ERR_INVALID_ARG;   // nowhere to append
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t q_bytes = static_cast<size_t>(N) * Hq * D * 2, kv_bytes = static_cast<size_t>(N) * Hkv * D * 2;
  if (cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(k_new_dev, k_new_host, kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(v_new_dev, v_new_host, kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  st = attn_kv_append(k_new_dev, v_new_dev, k_pool, v_pool, page_table, seq_lens, page_size, N, Hkv, 1, D,
                      num_pages, max_pages, stream);
  if (st != ATTN_OK) return st;
  st = attn_decode_paged(q_dev, k_pool, v_pool, page_table, seq_lens, page_size, N, Hq, Hkv, D, num_pages,
                         max_pages, max_seq_len, scale, window, workspace, workspace_bytes, out_dev, stream);
  if (st != ATTN_OK) return st;
  return cudaMemcpyAsync(out_host, out_dev, q_bytes, cudaMemcpyDeviceToHost, s) == cudaSuccess ? ATTN_OK
                                                                                             : ATTN_ERR_CUDA;
}

attn_status_t attn_decode_paged_noalloc(const void* q, const void* k_pool, const void* v_pool,
                                        const int32_t* page_table, const int32_t* seq_lens, int page_size, int N,
                                        int Hq, int Hkv, int D, int num_pages, int max_pages, int max_seq_len,
                                        float scale, int window, void* out, attn_stream_t stream) {
  // Same checks as attn_decode_paged, with the library's fixed scratch as the workspace.
  if (N < 0 || Hq < 0 || D <= 0 || max_seq_len < 0 || page_size <= 0) return ATTN_ERR_INVALID_ARG;
  const size_t need = (N == 0 || Hq == 0) ? 0 : attn::decode_workspace_bytes(N, Hq, D, max_seq_len, page_size);
  if (need > attn::decode_scratch_capacity()) return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    scratch = attn::decode_scratch_address();
    if (scratch == nullptr) return ATTN_ERR_CUDA;
  }
  return attn_decode_paged(q, k_pool, v_pool, page_table, seq_lens, page_size, N, Hq, Hkv, D, num_pages, max_pages,
                           max_seq_len, scale, window, scratch, attn::decode_scratch_capacity(), out, stream);
}

}  // extern "C"

namespace {

attn_status_t kv_append(const void* k_new, const void* v_new, void* k_pool, void* v_pool, const int32_t* page_table,
                        const int32_t* seq_lens, int page_size, int B, int Hkv, int S_new, int D, int num_pages,
                        int max_pages, attn_stream_t stream, bool fp8, float k_scale, float v_scale) {
  if (B < 0 || Hkv < 0 || S_new < 0 || D <= 0 || page_size <= 0 || num_pages < 0 || max_pages < 0)
    return ATTN_ERR_INVALID_ARG;
  if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale))
    return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hkv == 0 || S_new == 0) return ATTN_OK;
  if (k_new == nullptr || v_new == nullptr || k_pool == nullptr || v_pool == nullptr || page_table == nullptr ||
      seq_lens == nullptr || num_pages == 0 || max_pages == 0)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > 512 || page_size % 8 != 0) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hkv * S_new * (D / 8) > 0x7FFFFFFFLL) return ATTN_ERR_UNSUPPORTED;
  return from_cuda(attn::launch_kv_append(k_new, v_new, k_pool, v_pool, page_table, seq_lens, page_size, B, Hkv,
                                          S_new, D, num_pages, max_pages, attn::device_error_word(),
                                          reinterpret_cast<cudaStream_t>(stream), fp8, k_scale, v_scale));
}

}  // namespace

extern "C" {

attn_status_t attn_kv_append(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int32_t* page_table, const int32_t* seq_lens, int page_size, int B, int Hkv,
                             int S_new, int D, int num_pages, int max_pages, attn_stream_t stream) {
  return kv_append(k_new, v_new, k_pool, v_pool, page_table, seq_lens, page_size, B, Hkv, S_new, D, num_pages,
                   max_pages, stream, false, 1.f, 1.f);
}

attn_status_t attn_kv_append_fp8(const void* k_new, const void* v_new, uint8_t* k_pool, uint8_t* v_pool,
                                 const int32_t* page_table, const int32_t* seq_lens, int page_size, int B, int Hkv,
                                 int S_new, int D, int num_pages, int max_pages, float k_scale, float v_scale,
                                 attn_stream_t stream) {
  return kv_append(k_new, v_new, k_pool, v_pool, page_table, seq_lens, page_size, B, Hkv, S_new, D, num_pages,
                   max_pages, stream, true, k_scale, v_scale);
}

}  // extern "C"

namespace attn {
namespace {

// One thread waits, through the kernels' own bounded wait, for an mbarrier
// phase that nothing completes; the wait gives up after limit_ns and records
// a timeout in the error word, and the kernel returns normally.
__global__ void timeout_selftest_kernel(unsigned int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  abort_flag = 0;
  mbar_wait_for(&bar, 0, &abort_flag, err, limit_ns);
}

}  // namespace
}  // namespace attn

extern "C" {

attn_status_t attn_selftest_wait_timeout(int limit_ms, attn_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 1000) return ATTN_ERR_INVALID_ARG;
  unsigned int* err = attn::device_error_word();
  if (err == nullptr) return ATTN_ERR_CUDA;
  attn::timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      err, static_cast<unsigned long long>(limit_ms) * 1000000ull);
  return from_cuda(cudaGetLastError());
}

attn_status_t attn_device_status(int clear) {
  unsigned int* addr = attn::device_error_word();
  if (addr == nullptr) return ATTN_ERR_CUDA;
  unsigned int word = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpy(&word, addr, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpy(addr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (word & ATTN_ERRBIT_TIMEOUT) return ATTN_ERR_TIMEOUT;
  if (word & ATTN_ERRBIT_BADPAGE) return ATTN_ERR_BAD_PAGE;
  return ATTN_OK;
}

}  // extern "C"
