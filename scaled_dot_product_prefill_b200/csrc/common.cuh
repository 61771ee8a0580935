// common.cuh -- definitions shared by the kernels and the host API.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

// Upper bound of any single device-side wait (1 s).  No legitimate wait in
// these kernels lasts more than a few microseconds.
#ifndef ATTN_WAIT_NS
#define ATTN_WAIT_NS 1000000000ull
#endif

#define ATTN_ERRBIT_TIMEOUT 1u   // a bounded wait gave up
#define ATTN_ERRBIT_BADPAGE 2u   // a page-table entry outside the pool, or seq_len too long

namespace attn {

// Kernels receive a pointer to the per-device error word kept by the API
// translation unit and OR error bits into it.
__device__ __forceinline__ void record_error(unsigned int* err, unsigned int bit) {
  if (err != nullptr) atomicOr(err, bit);
}

// Device address of this device's error word (looked up once per device).
unsigned int* device_error_word();

// Programmatic dependent launch.  A kernel launched with launch_dependent()
// may be scheduled before the kernel ahead of it in the stream has finished,
// so that its launch and set-up overlap that kernel's tail.  Every such kernel
// calls grid_dependency_wait() before its first access to global memory: the
// wait returns once the preceding grid has completed and its writes are
// visible (at once when there is no such grid).  grid_dependents_may_start()
// lets the next kernel be scheduled before this one ends; it does not make
// this kernel's writes visible early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_may_start() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

// 3-D tensor map over [planes][rows][inner] elements of elem_bytes bytes (2: bf16, 1: bytes),
// boxes of box_inner x box_rows x 1, 128-byte swizzle.  False if the driver's encoder is
// unavailable or rejects the map.
bool make_tensor_map_3d(CUtensorMap* m, const void* base, int elem_bytes, int inner, int rows, int planes,
                        int box_inner, int box_rows);

// Number of SMs of the current device (cached per device), 0 on error.
int sm_count();

// Write -inf to n floats (the log-sum-exp of rows with no visible key).
cudaError_t fill_neg_inf(float* p, size_t n, cudaStream_t stream);

// Host-side launchers (defined next to their kernels).
// lse (optional, may be null): [B, Hq, Sq] float, natural-log log-sum-exp of each row's scaled scores.
cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                              int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
                              unsigned int* err, cudaStream_t stream);
cudaError_t launch_prefill_tc_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                    const int32_t* seq_lens, int page_size, int B, int Hq, int Hkv, int Sq, int D,
                                    int num_pages, int max_pages, int max_seq_len, float scale, int causal,
                                    int window, void* out, float* lse, unsigned int* err, cudaStream_t stream);
cudaError_t launch_prefill_f32(const float* q, const float* k, const float* v, float* out, float* lse, int B,
                               int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
                               cudaStream_t stream);

struct DecodeGeometry {
  int split_tokens;   // keys per split (multiple of 64)
  int max_splits;     // splits per sequence for max_seq_len
};
DecodeGeometry decode_geometry(int N, int Hq, int D, int max_seq_len, int page_size);
size_t decode_workspace_bytes(int N, int Hq, int D, int max_seq_len, int page_size);
size_t decode_scratch_capacity();
void* decode_scratch_address();
cudaError_t launch_decode_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                const int32_t* seq_lens, int page_size, int N, int Hq, int Hkv, int D,
                                int num_pages, int max_pages, int max_seq_len, float scale, int window,
                                void* workspace, void* out, unsigned int* err, cudaStream_t stream,
                                bool fp8 = false, float k_scale = 1.f, float v_scale = 1.f);

// k_new/v_new [B, Hkv, S_new, D] -> pools [num_pages, Hkv, page_size, D] at positions seq_lens[b] - S_new + i.
cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int32_t* page_table, const int32_t* seq_lens, int page_size, int B, int Hkv,
                             int S_new, int D, int num_pages, int max_pages, unsigned int* err, cudaStream_t stream,
                             bool fp8 = false, float k_scale = 1.f, float v_scale = 1.f);

}  // namespace attn
