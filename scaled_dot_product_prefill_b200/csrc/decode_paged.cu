// decode_paged.cu -- one decode step over a paged KV cache (split-KV + combine).
//
// What is computed: for every sequence b and query head h (kv head
// g = h / G, G = Hq / Hkv), o = softmax(K_b q * scale) V_b over the keys
// [lo, L) of the sequence's cache, L = seq_lens[b], lo = max(0, L - window)
// (lo = 0 without a window).  Token t lives in physical page
// page_table[b][t / page_size] at slot t % page_size ("Attention From
// Scratch" README, section "Paged KV Cache": fixed-size pages, per-sequence
// page tables, one shared pool; "LLM core technology", section
// "PagedAttention").  The cache already holds the new token, so no causal
// mask is needed ("Taking LLMs apart (2)", section "KV cache").
//
// How: decode is bound by HBM bandwidth (every K/V byte is read once per kv
// head and used for 2*G flops), so the design goal is bytes in flight and
// no wasted reads; tensor cores play no part.
//
// * decode_split_kernel: grid (split, kv head, sequence).  Each CTA owns a
//   span of `split_tokens` keys; its four warps take interleaved 16-token
//   chunks.  A chunk of one kv head is 16 * D contiguous bf16 (4 KB at
//   D = 128) inside one page, so each warp fetches K and V chunks with two
//   bulk asynchronous copies into its own shared-memory ring and never
//   stalls on individual loads.  Page-table entries for the warp's chunks
//   are read once, one per lane, up front.  All G query heads of the group
//   are evaluated against each K/V element while it is in registers.
//   The online softmax keeps a reference maximum per head and only moves it
//   (rescaling the running sum and accumulator) when a score exceeds it by
//   more than 2^8 in probability, which leaves the result exact.  Each
//   split writes its normalised partial output and base-2 log-sum-exp.
// * decode_combine_kernel: one warp per (sequence, head) merges the splits,
//   weighting each by 2^(lse_s - max lse) ("Attention From Scratch"
//   README, section "Flash Attention": the pair (output, lse)).  The lanes
//   load 32 splits' log-sum-exps at once; for sequences of up to 16 splits
//   (no window) every log-sum-exp and partial output is loaded together with
//   the sequence length, in one round trip.  It is launched as a dependent
//   of the split pass, so its launch overlaps that kernel's tail.
#include <cmath>
#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <pthread.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kWarps = 4;       // warps per split CTA
constexpr int kChunk = 16;      // tokens per chunk (one bulk copy per K and per V)
constexpr float kTau = 8.0f;    // lazy-rescale threshold, log2 units
constexpr int kStages = 2;      // ring depth per warp: 16-token K+V chunks at D = 128 (twice as many at D = 64)
constexpr int kSplit = 1024;    // keys per split when the batch fills the GPU
constexpr int kMinBlocks = 3;   // CTAs per SM the register allocation aims for
// a warp's chunks of one split have their page-table entries in one lane each
static_assert(kSplit / (kChunk * kWarps) <= 32, "at most 32 chunks per warp and split");

struct DecodeParams {
  const __nv_bfloat16* q;
  const void* k_pool;   // bf16 or fp8 e4m3 codes, [num_pages, Hkv, page_size, D]
  const void* v_pool;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* ws_o;        // [N, Hq, max_splits, D]
  float* ws_lse;      // [N, Hq, max_splits]
  __nv_bfloat16* out; // [N, Hq, D]
  unsigned int* err;
  int page_size, Hq, Hkv, num_pages, max_pages, max_seq_len;
  int split_tokens, max_splits, window;
  float scale_log2;   // softmax scale (times the K scale for fp8) in log2 units
  float v_scale;      // output multiplier: the V scale for fp8, 1 for bf16
};

// 8 bf16 (one 16-byte load) as 4 packed fp32 pairs (element 2i in the low half).
__device__ __forceinline__ void bf16x8_to_f2(const uint4& u, uint64_t (&f)[4]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = f2_pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

// 8 fp8 e4m3 codes (one 8-byte load) as 4 packed fp32 pairs (element 2i in the
// low half): the hardware conversion to f16 pairs is exact, as is f16 -> f32.
__device__ __forceinline__ void fp8x8_to_f2(const uint2& u, uint64_t (&f)[4]) {
  const uint32_t w[2] = {u.x, u.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const unsigned short pair = static_cast<unsigned short>(w[i] >> (16 * h));
      uint32_t h2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
      float lo, hi;
      asm("{\n\t.reg .f16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
          : "=f"(lo), "=f"(hi)
          : "r"(h2));
      f[2 * i + h] = f2_pack(lo, hi);
    }
  }
}

// One lane's PIECES x 8 elements of token `tok`'s K row, for the scores, as
// packed fp32 pairs (piece p in f[4p, 4p+4)).  Lane c of a row (c < RQ) holds
// the 8-element groups c and c + RQ of the row (q_col), for bf16 and fp8 alike,
// so that both caches sum the same products in the same order.  Where eight
// (bf16) or sixteen (fp8) consecutive lanes would reach two rows through the
// same banks, the lanes of every other row read their second group first,
// and the two loads are put back in order in registers.
template <int D, bool FP8, int PIECES, int RQ>
__device__ __forceinline__ int q_col(int c, int piece) {
  return (c + piece * RQ) * 8;
}

template <int D, bool FP8, int PIECES, int RQ>
__device__ __forceinline__ void load_k_pieces(const uint8_t* base, int tok, int c, uint64_t (&f)[PIECES * 4]) {
  constexpr int EB = FP8 ? 1 : 2;
  const uint8_t* row = base + tok * D * EB;
  if constexpr (PIECES == 1) {
    if constexpr (FP8) {
      fp8x8_to_f2(*reinterpret_cast<const uint2*>(row + c * 8), f);
    } else {
      bf16x8_to_f2(*reinterpret_cast<const uint4*>(row + c * 16), f);
    }
  } else {
    const bool swap = (((tok * D * EB) >> 7) & 1) != 0;
    const int first = swap ? c + RQ : c, second = swap ? c : c + RQ;
    if constexpr (FP8) {
      const uint2 a = *reinterpret_cast<const uint2*>(row + first * 8);
      const uint2 b = *reinterpret_cast<const uint2*>(row + second * 8);
      uint64_t lo[4], hi[4];
      fp8x8_to_f2(swap ? b : a, lo);
      fp8x8_to_f2(swap ? a : b, hi);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[e] = lo[e];
        f[4 + e] = hi[e];
      }
    } else {
      const uint4 a = *reinterpret_cast<const uint4*>(row + first * 16);
      const uint4 b = *reinterpret_cast<const uint4*>(row + second * 16);
      uint64_t lo[4], hi[4];
      bf16x8_to_f2(swap ? b : a, lo);
      bf16x8_to_f2(swap ? a : b, hi);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[e] = lo[e];
        f[4 + e] = hi[e];
      }
    }
  }
}

// One lane's 8 elements of a V row from shared memory as packed fp32 pairs.
template <bool FP8>
__device__ __forceinline__ void load8_f2(const uint8_t* base, int idx, bool zero, uint64_t (&f)[4]) {
  if constexpr (FP8) {
    uint2 u = reinterpret_cast<const uint2*>(base)[idx];
    if (zero) u = make_uint2(0u, 0u);
    fp8x8_to_f2(u, f);
  } else {
    uint4 u = reinterpret_cast<const uint4*>(base)[idx];
    if (zero) u = make_uint4(0u, 0u, 0u, 0u);
    bf16x8_to_f2(u, f);
  }
}

// Sum NV per-lane values over groups of R lanes (lane bits below R) and
// leave each lane with max(1, NV / R) fully reduced values; `base` returns
// the original index of the lane's first value.
template <int NV, int R>
__device__ __forceinline__ void reduce_scatter(float (&v)[NV], int lane, int& base) {
  base = 0;
  int n = NV;
#pragma unroll
  for (int m = R / 2; m >= 1; m >>= 1) {
    if (n > 1) {
      const int half = n / 2;
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int j = 0; j < NV / 2; ++j) {
        if (j < half) {
          const float send = upper ? v[j] : v[half + j];
          const float keep = upper ? v[half + j] : v[j];
          v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      base += upper ? half : 0;
      n = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
}

// FP8: K and V are e4m3 codes (1 byte per element) instead of bf16.  Every lane
// handles 8 elements of a row either way, so the ring keeps its bytes and
// holds twice the chunks for fp8.
template <int D, bool FP8>
struct Geo {
  static constexpr int EB = FP8 ? 1 : 2;          // bytes per element
  static constexpr int R = D / 8;                 // P.V: lanes per token row (8 elements each)
  static constexpr int TPL = 32 / R;              // P.V: tokens per warp-wide load
  static constexpr int NL = kChunk / TPL;         // P.V: loads per chunk per lane
  static constexpr int CHUNK_BYTES = kChunk * D * EB;
  static constexpr int STAGES = ((D == 128) ? kStages : 2 * kStages) * (FP8 ? 2 : 1);
};

template <int D, int G, bool FP8>
struct SplitSmem {
  alignas(1024) uint8_t ring[kWarps][Geo<D, FP8>::STAGES][2][Geo<D, FP8>::CHUNK_BYTES];  // K then V
  alignas(16) float pbuf[kWarps][kChunk * G];     // p of the current chunk, [token][head]
  float wm[kWarps][G];                            // per-warp reference max (log2 units)
  float wl[kWarps][G];                            // per-warp running sum
  uint64_t full[kWarps][Geo<D, FP8>::STAGES];
  int stage_ok[kWarps][Geo<D, FP8>::STAGES];
};

// Groups of 8 query heads hold twice the accumulators: 2 CTAs per SM leave them 255 registers.
template <int D, int G, bool FP8>
__global__ void __launch_bounds__(kWarps * 32, (G >= 8) ? 2 : kMinBlocks)
    decode_split_kernel(const DecodeParams p) {
  using Gm = Geo<D, FP8>;
  constexpr int R = Gm::R, TPL = Gm::TPL, NL = Gm::NL, STAGES = Gm::STAGES;
  // Scores: with up to 4 heads per group a lane takes two 8-column pieces of
  // a K row, so a row spans half as many lanes and its dot products need one
  // fewer shuffle level; the q registers this costs do not fit for 8 heads.
  constexpr int PIECES = (G <= 4) ? 2 : 1;
  constexpr int RQ = R / PIECES;                   // lanes per K row for the scores
  constexpr int TPLQ = 32 / RQ;                    // tokens per warp-wide K load
  constexpr int NLQ = kChunk / TPLQ;               // K loads per chunk per lane
  constexpr int NV = NLQ * G;                      // partial dot products per lane per chunk
  constexpr int NF = (NV / RQ) > 0 ? (NV / RQ) : 1;  // scores held per lane after reduction
  constexpr int DUP = (NV >= RQ) ? 1 : RQ / NV;       // lanes sharing one score when NV < RQ
  extern __shared__ uint8_t smem_raw[];
  SplitSmem<D, G, FP8>& sm = *reinterpret_cast<SplitSmem<D, G, FP8>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // inputs may come from the kernel before (the append of the new token)
  grid_dependency_wait();
  // once every split CTA has started, the combine may be scheduled into the SMs this grid frees
  grid_dependents_may_start();
  int L = p.seq_lens[b];
  if (L > p.max_seq_len || L > p.max_pages * p.page_size) {
    if (threadIdx.x == 0 && s == 0) record_error(p.err, ATTN_ERRBIT_BADPAGE);
    L = min(L, min(p.max_seq_len, p.max_pages * p.page_size));
  }
  if (L <= 0) return;
  const int lo = (p.window > 0) ? max(0, L - p.window) : 0;
  if (s < lo / p.split_tokens || s > (L - 1) / p.split_tokens) return;  // split holds no visible key

  const int t_begin = max(s * p.split_tokens, lo);
  const int t_end = min((s + 1) * p.split_tokens, L);
  const int c_begin = t_begin / kChunk;
  const int c_end = (t_end + kChunk - 1) / kChunk;
  // chunks of this warp: c_begin + warp + kWarps * i
  const int n_my = (c_end - c_begin - warp + kWarps - 1) / kWarps;  // may be <= 0

  if (threadIdx.x < kWarps * STAGES) {
    mbar_init(&sm.full[threadIdx.x / STAGES][threadIdx.x % STAGES], 1);
  }
  fence_mbar_init();
  __syncthreads();

  const size_t head_stride = static_cast<size_t>(p.page_size) * D;  // elements per (page, head)
  // lane i holds the physical page of the warp's i-th chunk
  int my_page = -1;
  if (lane < n_my) {
    const int t0 = (c_begin + warp + kWarps * lane) * kChunk;
    my_page = p.page_table[static_cast<size_t>(b) * p.max_pages + t0 / p.page_size];
  }

  auto issue = [&](int i) {  // whole warp calls; lane 0 issues chunk i into stage i % STAGES
    const int phys = __shfl_sync(0xffffffffu, my_page, i);
    if (lane == 0) {
      const int st = i % STAGES;
      uint64_t* bar = &sm.full[warp][st];
      if (phys < 0 || phys >= p.num_pages) {
        record_error(p.err, ATTN_ERRBIT_BADPAGE);
        sm.stage_ok[warp][st] = 0;
        mbar_arrive(bar);
      } else {
        sm.stage_ok[warp][st] = 1;
        const int t0 = (c_begin + warp + kWarps * i) * kChunk;
        const size_t off = (static_cast<size_t>(phys) * p.Hkv + g) * head_stride +
                           static_cast<size_t>(t0 % p.page_size) * D;
        mbar_arrive_expect_tx(bar, 2 * Gm::CHUNK_BYTES);
        bulk_load(sm.ring[warp][st][0], static_cast<const uint8_t*>(p.k_pool) + off * Gm::EB, Gm::CHUNK_BYTES, bar);
        bulk_load(sm.ring[warp][st][1], static_cast<const uint8_t*>(p.v_pool) + off * Gm::EB, Gm::CHUNK_BYTES, bar);
      }
    }
  };

  const int n_pro = min(n_my, STAGES);
  for (int i = 0; i < n_pro; ++i) issue(i);

  // query of the G heads of this group, the score phase's columns of this
  // lane, pre-scaled to log2 units; d0: the P.V phase's 8 columns
  const int d0 = (lane % R) * 8;
  // (packed fp32 pairs: the dot products and the P.V accumulation run as f32x2 FMAs)
  uint64_t q2[G][PIECES * 4];
  const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
#pragma unroll
    for (int pc = 0; pc < PIECES; ++pc) {
      const uint4 u = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * p.Hq + g * G + hh) * D +
                                                      q_col<D, FP8, PIECES, RQ>(lane % RQ, pc));
      uint64_t a[4];
      bf16x8_to_f2(u, a);
#pragma unroll
      for (int e = 0; e < 4; ++e) q2[hh][4 * pc + e] = f2_mul(a[e], sc2);
    }
  }

  float m_ref[G], l_part[G];
  uint64_t acc2[G][4];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    m_ref[hh] = -INFINITY;
    l_part[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc2[hh][e] = f2_pack(0.f, 0.f);
  }

  bool ok_all = true;
  for (int i = 0; i < n_my; ++i) {
    const int st = i % STAGES;
    if (!mbar_wait(&sm.full[warp][st], (i / STAGES) & 1, nullptr, p.err)) {
      // give the copies still in flight a bounded chance to land before the ring is reused
      for (int k = i + 1; k < min(n_my, i + STAGES); ++k)
        mbar_wait(&sm.full[warp][k % STAGES], (k / STAGES) & 1, nullptr, p.err);
      ok_all = false;
      break;
    }
    const int chunk_t0 = (c_begin + warp + kWarps * i) * kChunk;
    const bool stage_ok = sm.stage_ok[warp][st] != 0;
    const bool full = stage_ok && chunk_t0 >= lo && chunk_t0 + kChunk <= L;
    const uint8_t* sk = sm.ring[warp][st][0];
    const uint8_t* sv = sm.ring[warp][st][1];

    // ---- scores: partial dot products over my columns, then reduce over the row's RQ lanes
    float part[NV];
#pragma unroll
    for (int l = 0; l < NLQ; ++l) {
      uint64_t k2[PIECES * 4];
      load_k_pieces<D, FP8, PIECES, RQ>(sk, l * TPLQ + lane / RQ, lane % RQ, k2);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        uint64_t a = f2_mul(q2[hh][0], k2[0]);
#pragma unroll
        for (int e = 1; e < PIECES * 4; ++e) a = f2_fma(q2[hh][e], k2[e], a);
        float x0, x1;
        f2_unpack(a, x0, x1);
        part[l * G + hh] = x0 + x1;
      }
    }
    int base;
    reduce_scatter<NV, RQ>(part, lane, base);

    // my NF scores: index idx = base + j  ->  load l = idx / G, head idx % G, token l*TPLQ + lane/RQ
    float sc[NF];
    int hd[NF];
    bool any_up = false;
#pragma unroll
    for (int j = 0; j < NF; ++j) {
      const int idx = base + j;
      const int tok = (idx / G) * TPLQ + lane / RQ;
      const int t = chunk_t0 + tok;
      const bool vis = stage_ok && t >= lo && t < L;
      hd[j] = idx % G;
      sc[j] = vis ? part[j] : -INFINITY;
      float mr = m_ref[0];
#pragma unroll
      for (int hh = 1; hh < G; ++hh) mr = (hd[j] == hh) ? m_ref[hh] : mr;
      any_up |= sc[j] > mr + kTau;
    }
    if (__any_sync(0xffffffffu, any_up)) {
      // move the reference maxima to the new per-head maxima of this chunk
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < NF; ++j) mx = (hd[j] == hh) ? fmaxf(mx, sc[j]) : mx;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (mx > m_ref[hh] + kTau) {
          const float alpha = (m_ref[hh] == -INFINITY) ? 0.f : ex2(m_ref[hh] - mx);
          l_part[hh] *= alpha;
          const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc2[hh][e] = f2_mul(acc2[hh][e], a2);
          m_ref[hh] = mx;
        }
      }
    }
    // probabilities relative to the reference maxima, shared through shared memory
    float* pb = sm.pbuf[warp];
#pragma unroll
    for (int j = 0; j < NF; ++j) {
      float mr = m_ref[0];
#pragma unroll
      for (int hh = 1; hh < G; ++hh) mr = (hd[j] == hh) ? m_ref[hh] : mr;
      const float pr = (sc[j] == -INFINITY) ? 0.f : ex2(sc[j] - mr);
      // with fewer values than lanes, DUP neighbouring lanes hold the same score: count it once
      const bool counted = (lane & (DUP - 1)) == 0;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) l_part[hh] += (hd[j] == hh && counted) ? pr : 0.f;
      const int idx = base + j;
      pb[((idx / G) * TPLQ + lane / RQ) * G + (idx % G)] = pr;
    }
    __syncwarp();

    // ---- P.V over my 8 columns and my tokens
#pragma unroll
    for (int l = 0; l < NL; ++l) {
      const int tok = l * TPL + lane / R;
      bool zero = false;
      if (!full) {
        const int t = chunk_t0 + tok;
        zero = !(stage_ok && t >= lo && t < L);   // poisoned slots stay out
      }
      uint64_t v2[4];
      load8_f2<FP8>(sv, l * 32 + lane, zero, v2);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float pr = pb[tok * G + hh];
        const uint64_t pp = f2_pack(pr, pr);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc2[hh][e] = f2_fma(pp, v2[e], acc2[hh][e]);
      }
    }
    __syncwarp();
    fence_proxy_async_smem();
    if (i + STAGES < n_my) issue(i + STAGES);
  }

  // ---- per-warp totals: accumulators over the TPL token groups, sums over all lanes
  float acc[G][8];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int e = 0; e < 4; ++e) f2_unpack(acc2[hh][e], acc[hh][2 * e], acc[hh][2 * e + 1]);
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
#pragma unroll
    for (int o = R; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[hh][e] += __shfl_xor_sync(0xffffffffu, acc[hh][e], o);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l_part[hh] += __shfl_xor_sync(0xffffffffu, l_part[hh], o);
  }
  if (!ok_all) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) m_ref[hh] = -INFINITY;   // contribute nothing
  }
  // every stage this warp issued has been waited on, so the ring can be reused
  __syncthreads();
  float* wacc = reinterpret_cast<float*>(&sm.ring[0][0][0][0]);   // [kWarps][G][D]
  if (lane < R) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int e = 0; e < 8; ++e) wacc[(warp * G + hh) * D + d0 + e] = acc[hh][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      sm.wm[warp][hh] = m_ref[hh];
      sm.wl[warp][hh] = l_part[hh];
    }
  }
  __syncthreads();

  // ---- merge the warps and write this split's partial output and lse
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int hh = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.wm[w][hh]);
    float o = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = (sm.wm[w][hh] == -INFINITY) ? 0.f : ex2(sm.wm[w][hh] - M);
        o += f * wacc[(w * G + hh) * D + d];
        lsum += f * sm.wl[w][hh];
      }
    }
    const size_t row = (static_cast<size_t>(b) * p.Hq + g * G + hh) * p.max_splits + s;
    p.ws_o[row * D + d] = (lsum > 0.f) ? o / lsum : 0.f;
    if (d == 0) p.ws_lse[row] = (lsum > 0.f) ? M + log2f(lsum) : -INFINITY;
  }
}

template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p, int N) {
  constexpr int PER = D / 32;    // output columns per lane: 4 (one 16-byte load) or 2 (8 bytes)
  constexpr int SPEC = 16;       // splits whose partials are loaded before the sequence length is known
  using VecT = typename std::conditional<PER == 4, float4, float2>::type;
  const int warp_global = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  grid_dependency_wait();   // the split pass's partials
  if (warp_global >= N * p.Hq) return;
  const int b = warp_global / p.Hq;
  const size_t rowbase = static_cast<size_t>(warp_global) * p.max_splits;
  // Without a window a sequence of up to SPEC splits uses splits [0, s1]: their
  // log-sum-exps and partial outputs are loaded together with seq_lens, so the
  // common case costs one round trip to memory.  Rows past s1 hold data of
  // earlier calls (or none) and are never used.
  const int nspec = min(SPEC, p.max_splits);
  const float lse_spec = (lane < min(32, p.max_splits)) ? p.ws_lse[rowbase + lane] : -INFINITY;
  VecT vs[SPEC];
#pragma unroll
  for (int k = 0; k < SPEC; ++k)
    if (k < nspec) vs[k] = *reinterpret_cast<const VecT*>(p.ws_o + (rowbase + k) * D + lane * PER);
  int L = p.seq_lens[b];
  L = min(L, min(p.max_seq_len, p.max_pages * p.page_size));
  __nv_bfloat16* op = p.out + static_cast<size_t>(warp_global) * D;
  float acc[PER];
#pragma unroll
  for (int t = 0; t < PER; ++t) acc[t] = 0.f;
  float wsum = 0.f;
  auto add = [&](float wk, const VecT& v) {
    acc[0] = fmaf(wk, v.x, acc[0]);
    acc[1] = fmaf(wk, v.y, acc[1]);
    if constexpr (PER == 4) {
      acc[2] = fmaf(wk, v.z, acc[2]);
      acc[3] = fmaf(wk, v.w, acc[3]);
    }
  };
  if (L > 0) {
    const int lo = (p.window > 0) ? max(0, L - p.window) : 0;
    const int s0 = lo / p.split_tokens, s1 = (L - 1) / p.split_tokens;
    if (s0 == 0 && s1 < nspec) {
      const float lse = (lane <= s1) ? lse_spec : -INFINITY;
      float M = lse;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      if (M != -INFINITY) {
        const float w = (lse == -INFINITY) ? 0.f : ex2(lse - M);   // lane k holds split k's weight
        wsum = w;
#pragma unroll
        for (int k = 0; k < SPEC; ++k) {
          const float wk = __shfl_sync(0xffffffffu, w, k);
          if (k <= s1) add(wk, vs[k]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
      }
    } else {
      // the splits' log-sum-exps, 32 at a time across the lanes, and their maximum
      float M = -INFINITY;
      for (int s = s0 + lane; s <= s1; s += 32) M = fmaxf(M, p.ws_lse[rowbase + s]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      if (M != -INFINITY) {
        for (int base = s0; base <= s1; base += 32) {
          const int s = base + lane;
          const float lse = (s <= s1) ? p.ws_lse[rowbase + s] : -INFINITY;
          const float w = (lse == -INFINITY) ? 0.f : ex2(lse - M);   // lane k holds split base + k's weight
          wsum += w;
          const int cnt = min(32, s1 - base + 1);
          // independent loads of several splits' partial outputs in flight
#pragma unroll 8
          for (int k = 0; k < cnt; ++k) {
            const float wk = __shfl_sync(0xffffffffu, w, k);
            add(wk, *reinterpret_cast<const VecT*>(p.ws_o + (rowbase + base + k) * D + lane * PER));
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
      }
    }
  }
  const float inv = (wsum > 0.f) ? p.v_scale / wsum : 0.f;
#pragma unroll
  for (int t = 0; t < PER; t += 2) {
    __nv_bfloat162 v2 = __floats2bfloat162_rn(acc[t] * inv, acc[t + 1] * inv);
    *reinterpret_cast<__nv_bfloat162*>(op + lane * PER + t) = v2;
  }
}

template <int D, int G, bool FP8>
cudaError_t launch_split(const DecodeParams& p, int N, cudaStream_t stream) {
  const size_t smem = sizeof(SplitSmem<D, G, FP8>) + 1024;
  auto kern = decode_split_kernel<D, G, FP8>;
  // the shared-memory limit is set once per device (a runtime call per launch costs host time)
  constexpr int kMaxDevices = 64;
  static int ready[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE) != 1) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
  }
  dim3 grid(p.max_splits, p.Hkv, N);
  return launch_dependent(kern, grid, dim3(kWarps * 32), smem, stream, p);
}

}  // namespace

DecodeGeometry decode_geometry(int N, int Hq, int D, int max_seq_len, int page_size) {
  (void)Hq;
  (void)D;
  (void)page_size;
  DecodeGeometry g{};
  // kSplit keys per split (16 chunks per warp at 1024), which amortises
  // each CTA's set-up (barriers, page-table reads, q) and its partial-output
  // write; shorter splits when the batch has too few (sequence, split) pairs
  // to fill the GPU.  On the 64-sequence, 512-8192-token workload splits of
  // 256, 512, 768, 1024, 1536 and 2048 keys took 0.259, 0.220, 0.216, 0.212,
  // 0.216 and 0.220 ms.
  int split = kSplit;
  const long long units = static_cast<long long>(N);
  while (split > 64 && units * ((max_seq_len + split - 1) / split) < 512) split /= 2;
  g.split_tokens = split;
  g.max_splits = max_seq_len > 0 ? (max_seq_len + split - 1) / split : 1;
  return g;
}

size_t decode_workspace_bytes(int N, int Hq, int D, int max_seq_len, int page_size) {
  const DecodeGeometry g = decode_geometry(N, Hq, D, max_seq_len, page_size);
  const size_t rows = static_cast<size_t>(N) * Hq * g.max_splits;
  const size_t o_bytes = rows * D * sizeof(float);
  const size_t lse_bytes = ((rows * sizeof(float)) + 255) & ~static_cast<size_t>(255);
  return o_bytes + lse_bytes;
}

cudaError_t launch_decode_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                const int32_t* seq_lens, int page_size, int N, int Hq, int Hkv, int D,
                                int num_pages, int max_pages, int max_seq_len, float scale, int window,
                                void* workspace, void* out, unsigned int* err, cudaStream_t stream, bool fp8,
                                float k_scale, float v_scale) {
  const DecodeGeometry geo = decode_geometry(N, Hq, D, max_seq_len, page_size);
  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pool = k_pool;
  p.v_pool = v_pool;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  const size_t rows = static_cast<size_t>(N) * Hq * geo.max_splits;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + rows * D * sizeof(float));
  p.err = err;
  p.page_size = page_size;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.num_pages = num_pages;
  p.max_pages = max_pages;
  p.max_seq_len = max_seq_len;
  p.split_tokens = geo.split_tokens;
  p.max_splits = geo.max_splits;
  p.window = window;
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  p.v_scale = v_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  const int G = Hq / Hkv;
  cudaError_t e = cudaErrorInvalidValue;
#define ATTN_DECODE_CASE(DD, GG)                                        \
  if (D == DD && G == GG)                                               \
    e = fp8 ? launch_split<DD, GG, true>(p, N, stream) : launch_split<DD, GG, false>(p, N, stream);
  ATTN_DECODE_CASE(128, 1) ATTN_DECODE_CASE(128, 2) ATTN_DECODE_CASE(128, 4) ATTN_DECODE_CASE(128, 8)
  ATTN_DECODE_CASE(64, 1) ATTN_DECODE_CASE(64, 2) ATTN_DECODE_CASE(64, 4) ATTN_DECODE_CASE(64, 8)
#undef ATTN_DECODE_CASE
  if (e != cudaSuccess) return e;
  const int warps = N * Hq;
  const dim3 grid((warps + 3) / 4);
  if (D == 128) return launch_dependent(decode_combine_kernel<128>, grid, dim3(128), 0, stream, p, N);
  return launch_dependent(decode_combine_kernel<64>, grid, dim3(128), 0, stream, p, N);
}


// ---------------------------------------------------------------------------
// Fixed scratch for attn_decode_paged_noalloc.
//
// Some callers cannot allocate device memory at the point where they decode:
// code behind an interface that has no workspace argument (a plugin ABI fixed
// by a host framework), or a serving loop whose device memory is planned once
// at start-up and where a cudaMalloc, which may also synchronise the device,
// is not allowed.  For them the split-KV partials live in this file-scope
// array instead of a caller-provided workspace.  Every GPU that loads the
// library holds these kDecodeScratchBytes until the process exits.  All calls
// share the array: calls that overlap on the GPU (two streams, or two
// threads) race on it.  Nothing in it needs to start at zero: each call
// writes every partial output and log-sum-exp it later reads.
constexpr size_t kDecodeScratchBytes = size_t(32) << 20;   // 32 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

size_t decode_scratch_capacity() { return kDecodeScratchBytes; }

// Device address of g_decode_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, and cached.
void* decode_scratch_address() {
  constexpr int kMaxDevices = 64;
  static void* addr[kMaxDevices] = {};
  static pthread_mutex_t mu = PTHREAD_MUTEX_INITIALIZER;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  pthread_mutex_lock(&mu);
  if (addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) == cudaSuccess) addr[dev] = ptr;
  }
  void* a = addr[dev];
  pthread_mutex_unlock(&mu);
  return a;
}

}  // namespace attn
