// kv_append.cu -- write new tokens' keys and values into the paged KV cache.
//
// The kv-cache step of "Taking LLMs apart (2): attention by hand" (section
// "KV cache") stores the new token's k and v before that step's attention;
// the "Attention From Scratch" README (section "Paged KV Cache") keeps the
// cache in fixed-size pages located through a per-sequence page table.  This
// kernel is that store for a chunk of S_new tokens of each of B sequences:
// token i of sequence b lands at position seq_lens[b] - S_new + i, i.e. in page
// page_table[b][pos / page_size], slot pos % page_size.
//
// It is a pure copy and bound by HBM: 2 * B * Hkv * S_new * D * 2 bytes read
// and as many written.  A thread moves 16-byte pieces of (token, head) rows of
// K and the same pieces of V; consecutive threads cover consecutive pieces of
// a row, so the reads and (within a row) the writes coalesce.  A thread takes
// ATTN_APPEND_UNROLL pieces per pass and issues all their loads, page-table
// lookups included, before its stores.  One piece per pass is the default: on
// B200, 537 MB copies run at the same rate with 1, 2 or 4 pieces (about 83 %
// of a plain device copy), while at serving sizes (a 50 MB prefill chunk, a
// 0.5 MB decode step) more pieces per thread meant fewer blocks and less
// bandwidth.
#include "common.cuh"

namespace attn {
namespace {

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

#ifndef ATTN_APPEND_UNROLL
#define ATTN_APPEND_UNROLL 1
#endif
constexpr int kThreads = 256;
constexpr int kUnroll = ATTN_APPEND_UNROLL;   // pieces per thread per pass, all loads issued before any store

// 8 bf16 -> 8 FP8 E4M3 codes of x * inv_scale, rounded to nearest even and
// saturated at +-448 (cvt.rn.satfinite); element 0 lands in the lowest byte.
__device__ __forceinline__ uint2 quantize8_e4m3(const uint4& u, float inv_scale) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x0 = __uint_as_float(w[i] << 16) * inv_scale;
    const float x1 = __uint_as_float(w[i] & 0xFFFF0000u) * inv_scale;
    unsigned short pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(x1), "f"(x0));   // x1 high, x0 low
    out[i >> 1] |= static_cast<uint32_t>(pair) << (16 * (i & 1));
  }
  return make_uint2(out[0], out[1]);
}

// FP8: the pools hold E4M3 codes and each 16-byte piece of a bf16 row becomes
// 8 bytes of codes (k * k_inv, v * v_inv).
template <bool FP8>
__global__ void __launch_bounds__(kThreads) kv_append_kernel(const uint4* __restrict__ k_new,
                                                             const uint4* __restrict__ v_new,
                                                             void* __restrict__ k_pool, void* __restrict__ v_pool,
                                                             const int32_t* __restrict__ page_table,
                                                             const int32_t* __restrict__ seq_lens, int page_size,
                                                             int B, int Hkv, int S_new, int pieces, int num_pages,
                                                             int max_pages, unsigned int* err, float k_inv,
                                                             float v_inv) {
  grid_dependency_wait();   // the pools may still be read by the kernel before
  grid_dependents_may_start();
  const unsigned int total = static_cast<unsigned int>(B) * Hkv * S_new * pieces;
  const unsigned int pass = gridDim.x * kThreads * kUnroll;
  for (unsigned int base = blockIdx.x * kThreads * kUnroll + threadIdx.x; base < total; base += pass) {
    uint4 kv[kUnroll], vv[kUnroll];
    size_t dst[kUnroll];
    bool ok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      // t enumerates [B, Hkv, S_new, pieces] in layout order: it is also the source index
      const unsigned int t = base + u * kThreads;
      ok[u] = t < total;
      if (!ok[u]) continue;
      kv[u] = ld_stream(k_new + t);
      vv[u] = ld_stream(v_new + t);
      unsigned int r = t / pieces;
      const int c = static_cast<int>(t - r * pieces);
      const int i = static_cast<int>(r % S_new);
      r /= S_new;
      const int g = static_cast<int>(r % Hkv);
      const int b = static_cast<int>(r / Hkv);
      const int pos = seq_lens[b] - S_new + i;
      if (pos < 0) {   // the cache is shorter than the chunk: this token has no slot
        ok[u] = false;
        continue;
      }
      const int pg = pos / page_size;
      const int ph = (pg < max_pages) ? page_table[static_cast<size_t>(b) * max_pages + pg] : -1;
      if (ph < 0 || ph >= num_pages) {
        if (c == 0) record_error(err, ATTN_ERRBIT_BADPAGE);
        ok[u] = false;
        continue;
      }
      dst[u] = ((static_cast<size_t>(ph) * Hkv + g) * page_size + (pos - pg * page_size)) * pieces + c;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!ok[u]) continue;
      if constexpr (FP8) {
        static_cast<uint2*>(k_pool)[dst[u]] = quantize8_e4m3(kv[u], k_inv);
        static_cast<uint2*>(v_pool)[dst[u]] = quantize8_e4m3(vv[u], v_inv);
      } else {
        static_cast<uint4*>(k_pool)[dst[u]] = kv[u];
        static_cast<uint4*>(v_pool)[dst[u]] = vv[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int32_t* page_table, const int32_t* seq_lens, int page_size, int B, int Hkv,
                             int S_new, int D, int num_pages, int max_pages, unsigned int* err, cudaStream_t stream,
                             bool fp8, float k_scale, float v_scale) {
  static int sms[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int n_sm = (dev < 64 && sms[dev] > 0) ? sms[dev] : 148;
  const int pieces = D / 8;
  const long long total = static_cast<long long>(B) * Hkv * S_new * pieces;
  // one pass of resident blocks (8 x 256 threads per SM) covers up to 8 * n_sm * 256 * kUnroll pieces
  const long long want = (total + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  const int grid = static_cast<int>(want < 8LL * n_sm ? want : 8LL * n_sm);
  auto kern = fp8 ? kv_append_kernel<true> : kv_append_kernel<false>;
  return launch_dependent(kern, dim3(grid), dim3(kThreads), 0, stream, static_cast<const uint4*>(k_new),
                          static_cast<const uint4*>(v_new), k_pool, v_pool, page_table, seq_lens, page_size, B, Hkv,
                          S_new, pieces, num_pages, max_pages, err, 1.f / k_scale, 1.f / v_scale);
}

}  // namespace attn
