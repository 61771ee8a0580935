// prefill_f32.cu -- fp32 tiled attention on the CUDA cores (FFMA, no TF32).
//
// Same operation and masks as the bf16 tensor-core prefill, for inputs that
// must match a float64 evaluation to ~1e-5.  One warp owns one query row;
// the four warps of a CTA take four consecutive rows of one (batch, head)
// and share each 32-key tile of K and V staged in shared memory.  The
// softmax is the online form ("Attention From Scratch" README, section
// "Flash Attention": running maximum and running sum, earlier partial
// results rescaled when the maximum grows), evaluated in base 2 with the
// scale folded into the query: exp(x) = exp2(x * log2 e).
#include <cmath>
#include <cstdint>

#include "common.cuh"

namespace attn {
namespace {

constexpr int kRows = 4;      // query rows (warps) per CTA
constexpr int kKeys = 32;     // keys per tile

template <int D>
__global__ void __launch_bounds__(kRows * 32) prefill_f32_kernel(const float* __restrict__ q,
                                                                  const float* __restrict__ k,
                                                                  const float* __restrict__ v,
                                                                  float* __restrict__ out,
                                                                  float* __restrict__ lse, int Hq, int Hkv,
                                                                  int Sq, int Skv, float scale_log2,
                                                                  int causal, int window) {
  constexpr int PER = D / 32;            // output columns per lane
  __shared__ float sK[kKeys][D + 1];     // +1: lane j reads row j without bank conflicts
  __shared__ float sV[kKeys][D];
  __shared__ float sQ[kRows][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;             // b * Hq + h
  const int b = bh / Hq, h = bh % Hq;
  const int g = h / (Hq / Hkv);
  const int row0 = blockIdx.x * kRows;
  const int row = row0 + warp;
  const int off = Skv - Sq;

  const float* qp = q + (static_cast<size_t>(bh) * Sq) * D;
  const float* kp = k + (static_cast<size_t>(b) * Hkv + g) * static_cast<size_t>(Skv) * D;
  const float* vp = v + (static_cast<size_t>(b) * Hkv + g) * static_cast<size_t>(Skv) * D;

  for (int i = threadIdx.x; i < kRows * D; i += blockDim.x) {
    const int r = row0 + i / D;
    sQ[i / D][i % D] = (r < Sq) ? qp[static_cast<size_t>(r) * D + (i % D)] * scale_log2 : 0.f;
  }

  // key range of this CTA's rows: union over its (up to) kRows rows
  const int last_row = min(row0 + kRows, Sq) - 1;
  int k_lo = 0, k_hi = Skv;
  if (causal) {
    k_hi = min(Skv, last_row + off + 1);
    if (window > 0) k_lo = max(0, row0 + off - window + 1);
  }
  // this warp's own visible range [my_lo, my_hi)
  int my_lo = 0, my_hi = Skv;
  if (causal) {
    my_hi = min(Skv, row + off + 1);
    my_lo = (window > 0) ? max(0, row + off - window + 1) : 0;
  }

  float m = -INFINITY, l = 0.f;
  float acc[PER];
#pragma unroll
  for (int t = 0; t < PER; ++t) acc[t] = 0.f;

  for (int kt = (k_lo / kKeys) * kKeys; kt < k_hi; kt += kKeys) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKeys * D; i += blockDim.x) {
      const int j = kt + i / D;
      const bool in = j < Skv;
      sK[i / D][i % D] = in ? kp[static_cast<size_t>(j) * D + (i % D)] : 0.f;
      sV[i / D][i % D] = in ? vp[static_cast<size_t>(j) * D + (i % D)] : 0.f;
    }
    __syncthreads();

    const int j = kt + lane;
    float s = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) s = fmaf(sQ[warp][d], sK[lane][d], s);
    const bool vis = (row < Sq) && (j >= my_lo) && (j < my_hi);
    s = vis ? s : -INFINITY;

    float mt = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
    const float m_new = fmaxf(m, mt);
    const float base = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - base);
    const float p = vis ? exp2f(s - base) : 0.f;
    float ps = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * alpha + ps;
    m = m_new;
#pragma unroll
    for (int t = 0; t < PER; ++t) acc[t] *= alpha;
#pragma unroll 8
    for (int jj = 0; jj < kKeys; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
      for (int t = 0; t < PER; ++t) acc[t] = fmaf(pj, sV[jj][lane + 32 * t], acc[t]);
    }
  }

  if (row < Sq) {
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    if (lse != nullptr && lane == 0)   // log(sum_j exp(s_ij * scale)) = (m + log2 l) * ln 2
      lse[static_cast<size_t>(bh) * Sq + row] = (l > 0.f) ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    float* op = out + (static_cast<size_t>(bh) * Sq + row) * D;
#pragma unroll
    for (int t = 0; t < PER; ++t) op[lane + 32 * t] = acc[t] * inv;
  }
}

}  // namespace

cudaError_t launch_prefill_f32(const float* q, const float* k, const float* v, float* out, float* lse, int B,
                               int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
                               cudaStream_t stream) {
  const float scale_log2 = scale * 1.4426950408889634f;  // log2(e)
  dim3 grid((Sq + kRows - 1) / kRows, B * Hq);
  dim3 block(kRows * 32);
  if (D == 64) {
    prefill_f32_kernel<64><<<grid, block, 0, stream>>>(q, k, v, out, lse, Hq, Hkv, Sq, Skv, scale_log2, causal,
                                                       window);
  } else {
    prefill_f32_kernel<128><<<grid, block, 0, stream>>>(q, k, v, out, lse, Hq, Hkv, Sq, Skv, scale_log2, causal,
                                                        window);
  }
  return cudaGetLastError();
}

}  // namespace attn
