// decode_tc.cu -- the split pass of one paged decode step, both contractions on the tensor cores.
//
// What is computed: for sequence b, kv head g and one span ("split") of the
// keys the step reads, the attention of the G = Hq / Hkv query heads of the
// group over the visible keys of the span: the normalised partial output and
// its base-2 log-sum-exp.  The combine kernel of decode_paged.cu merges the
// splits.  Token t of sequence b lives in page page_table[b][t / page_size]
// at slot t % page_size ("Attention From Scratch" README, section "Paged KV
// Cache"; "LLM core technology", section "PagedAttention"); the cache holds
// the new token already ("Taking LLMs apart (2)", section "KV cache").
//
// How.  The step streams the cache once and is bound by HBM.  Done on CUDA
// cores, the 4 G D flops per key cost tens of warp-instructions per (key, kv
// head), so the SMs spend their issue slots on arithmetic instead of keeping
// loads in flight.  Here the G heads of a group become the N dimension of
// tensor-core products, padded to 16, the smallest N at M = 128:
//   S^T = K Q^T  M = 128 keys, N = 16, K = D.  A = the K tile, B = the
//                group's queries (rows past G are ignored).
//   O  += P V    M = 128 rows, of which the first G are the heads, N = D,
//                K = 128 keys.  A = P in shared memory (rows G..127 stay
//                zero), B = the V tile read MN-major, as in the prefill.
// The kernel is persistent: an item is (sequence, kv head, split of
// split_tokens keys), and CTA c takes items c, c + grid, ...  Each CTA has 9
// warps:
//   warps 0-3  softmax: thread t owns key t of the current 128-key tile (its
//              TMEM lane of S^T); per-head tile maxima are reduced across
//              the 128 threads, the reference maximum moves only when a
//              score exceeds it by 2^8 (exact: the final normalisation uses
//              the same reference), and each thread writes its key's column
//              of P.  Warp 0 also rescales and reads out O (TMEM lanes 0..G-1).
//   warps 4-7  loaders: warp 4 + s fills ring slot s (K and V tiles
//              alternate through the slots) with 16-byte cp.async copies that
//              land directly in the 128-byte-swizzled layout the MMA reads,
//              looking pages up in a page-table row read one item ahead.
//              Keys outside the item are zero-filled without a memory read.
//              Warp 4 also loads each item's 16 query rows by TMA.
//   warp 8     MMA issuer (one thread) and tensor-memory owner.
// A page of one kv head holds 16 rows of D bf16 at most 16-row granularity,
// so a 128-key tile gathers 8 or more pages; the swizzled layout needs every
// row's 16-byte chunks permuted, which the cp.async copies do for free while
// a tensor copy would need one 2 KB box per (page, 64 columns).  A loader warp
// waits for its own copies, fences them to the async proxy (the tensor cores
// read them) and arrives on its slot's barrier, so that no fence waits for
// another tile's copies and four tiles stay in flight.
// Per tile j the MMA thread issues S^T(j+1) before O += P(j) V(j), so the
// next tile's scores are ready when the softmax finishes the current one.  S^T
// and P are double-buffered, and so is O, so that one item's read-out
// overlaps the next item's first products.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kBT = 128;          // keys per tile
constexpr int kNH = 16;           // heads of a group, padded: the N of the score product
constexpr int kKSlots = 2;        // K ring: consumed by the S^T issuer a tile ahead of V
constexpr int kVSlots = 3;        // V ring: a slot is held until its P V product completes
constexpr int kSlots = kKSlots + kVSlots;
constexpr int kBox = 16;          // rows per page box (every supported page size is a multiple)
// warps 0-3 softmax (one per SM sub-partition), warp 4 the S^T issuer and
// tensor-memory owner, warp 5 the P V issuer, warps 6-9 the loaders
constexpr int kSWarp = 4;
constexpr int kPvWarp = 5;
constexpr int kLoadWarp0 = 6;
constexpr int kConvWarp0 = 10;    // 8-bit caches: warps 10-13 rewrite the codes as f16 in place
constexpr float kTau = 8.0f;      // lazy-rescale threshold, log2 units

template <int D>
struct TcCfg {
  static constexpr int KATOMS = D / 64;                 // 64-column (128-byte) swizzle atoms
  static constexpr int ATOM_BYTES = kBT * 128;          // one atom of a K or V tile
  static constexpr int TILE_BYTES = kBT * D * 2;
  static constexpr int Q_ATOM = kNH * 128;              // one atom of the queries (16 rows)
  static constexpr int Q_BYTES = kNH * D * 2;
  // P is the A operand of an M = 64 product: rows 0..G-1 are the heads, the
  // rest stay zero (the rows of O they make are never read)
  static constexpr int P_ATOM = 64 * 128;               // 64 keys of P (64 rows)
  static constexpr int P_BYTES = 64 * kBT * 2;
  // tensor memory: O buffer i at columns [D i, D i + D), S^T buffer i at [2 D + 16 i, 2 D + 16 i + 16)
  static constexpr uint32_t O_COL = 0;
  static constexpr uint32_t S_COL = 2 * D;
  static constexpr uint32_t TMEM_COLS = (S_COL + 2 * kNH <= 256) ? 256 : 512;
  static constexpr int BAR_BYTES = 512;                 // mbarriers, the TMEM address and the abort flag
  static constexpr int TAIL = BAR_BYTES + 1024;         // + reduction scratch
  static constexpr size_t SMEM = 1024 + 2 * Q_BYTES + 2 * P_BYTES + kSlots * TILE_BYTES + TAIL;
};

template <bool FP8>
constexpr int tc_threads() { return FP8 ? 448 : 320; }

struct TcParams {
  const void* k_pool;   // [num_pages, Hkv, page_size, D] bf16, or E4M3 codes
  const void* v_pool;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* ws_o;          // [N, Hq, max_splits, D]
  float* ws_lse;        // [N, Hq, max_splits]
  unsigned int* err;
  int Hq, Hkv, num_pages, max_pages, page_size, max_seq_len, window;
  int split_tokens, max_splits, n_items, q_rows;
  float scale_log2;
};

struct DItem {
  int b, g, s, t_begin, t_end, j0, nt;   // keys [t_begin, t_end) in tiles j0 .. j0 + nt - 1
};

// seq_lens of item k's sequence (0 past the last item).  Every role reads it
// one item ahead, so that the load's latency hides behind the current item.
__device__ __forceinline__ int item_len(const TcParams& p, int k) {
  return k < p.n_items ? p.seq_lens[k / (p.max_splits * p.Hkv)] : 0;
}

// Item k: split k % max_splits of kv head (k / max_splits) % Hkv of sequence
// k / (max_splits * Hkv), whose cache holds len keys.  nt = 0 if the split
// holds no visible key (or k is past the last item).
__device__ __forceinline__ DItem item_at(const TcParams& p, int k, int len) {
  DItem it;
  it.s = k % p.max_splits;
  const int r = k / p.max_splits;
  it.g = r % p.Hkv;
  it.b = r / p.Hkv;
  if (k >= p.n_items) len = 0;
  const int L = min(len, min(p.max_seq_len, p.max_pages * p.page_size));
  const int lo = (p.window > 0) ? max(0, L - p.window) : 0;
  it.t_begin = max(it.s * p.split_tokens, lo);
  it.t_end = min((it.s + 1) * p.split_tokens, L);
  it.j0 = it.t_begin / kBT;
  it.nt = (it.t_end > it.t_begin) ? (it.t_end - 1) / kBT + 1 - it.j0 : 0;
  return it;
}

// FP8: the pools hold E4M3 codes.  Their tiles arrive row-major in the upper
// half of a slot (one box of 16 rows x D bytes per page of one head); converter
// warps rewrite each in place as f16 (exact for every code) in the layout the
// MMA reads, and the queries and P are f16 as well, so the products run on f16
// operands.  The K scale is folded into the softmax scale, the V scale into the
// combine.
template <int D, int G, bool FP8>
__global__ void __launch_bounds__(tc_threads<FP8>(), 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const TcParams p) {
  using C = TcCfg<D>;
  constexpr int RAW_OFF = C::TILE_BYTES / 2;            // FP8: where a slot's codes land (row-major)
  static_assert(G >= 1 && G <= kNH, "group size");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                                   // [2][KATOMS][16 rows x 128 B]
  uint8_t* sP = sQ + 2 * C::Q_BYTES;                    // [2][2 atoms][64 rows x 128 B]
  uint8_t* sRing = sP + 2 * C::P_BYTES;                 // [kSlots][KATOMS][128 rows x 128 B]
  uint8_t* tail = sRing + kSlots * C::TILE_BYTES;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(tail);  // 2
  uint64_t* q_empty = q_full + 2;                       // 2
  uint64_t* full = q_empty + 2;                         // kSlots: K ring slots, then V ring slots
  uint64_t* empty = full + kSlots;                      // kSlots
  uint64_t* s_ready = empty + kSlots;                   // 2: S^T buffer written
  uint64_t* s_free = s_ready + 2;                       // 2: S^T buffer loaded by the softmax
  uint64_t* p_ready = s_free + 2;                       // 2: P buffer written
  uint64_t* p_free = p_ready + 2;                       // 2: P buffer read (and O current)
  uint64_t* o_full = p_free + 2;                        // 2: an item's last product into O buffer done
  uint64_t* o_free = o_full + 2;                        // 2: O buffer read out
  uint64_t* drain = o_free + 2;                         // 2: each issuer's products complete
  uint64_t* raw_full = drain + 2;                       // kSlots (FP8): a slot's codes have landed
  uint64_t* q_conv = raw_full + kSlots;                 // 2 (FP8): queries rewritten as f16
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_conv + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 + 2 + kSlots + kSlots + 6 * 2 + 2 + kSlots + 2) * 8 + 8 <= C::BAR_BYTES, "barrier area");
  float* red = reinterpret_cast<float*>(tail + C::BAR_BYTES);   // [2][4 warps][16]: tile maxima
  float* lred = red + 2 * 4 * kNH;                      // [4 warps][16]: row sums
  volatile int* okv = reinterpret_cast<volatile int*>(lred + 4 * kNH);   // [3][4 warps]: status at a barrier

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rounds = (p.n_items + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_ready[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_ready[i], 128);
      mbar_init(&p_free[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 128);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&full[s], FP8 ? 32 : 1);   // FP8: the converter warp's lanes; bf16: the TMA bytes
      mbar_init(&empty[s], 1);
      mbar_init(&raw_full[s], 1);
    }
    mbar_init(&q_conv[0], 32);
    mbar_init(&q_conv[1], 32);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp < 4) {
    // P rows G..127 stay zero for the whole kernel: the rows of O they make are never read
    uint4* z = reinterpret_cast<uint4*>(sP);
    for (int i = threadIdx.x; i < 2 * C::P_BYTES / 16; i += 128) z[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (warp == kSWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kLoadWarp0 && warp < kConvWarp0) {
    // ------------------------------------------------------------ loader warps 6-9
    // K tiles go to a ring of kKSlots slots, V tiles to a ring of kVSlots:
    // each ring has one consumer (the S^T issuer, the P V issuer) that takes
    // its tiles in order, and each slot one producer warp, so that no wait on
    // a slot's barrier can run a lap ahead of the slot.  Warps 6, 7 load the K
    // tiles t with t % kKSlots % 2 = 0, 1; warps 8, 9 the V tiles likewise.  A
    // tile is 8 x KATOMS page boxes of 16 rows x 64 columns, one per lane,
    // landing at their row offsets in the 128-byte-swizzled tile.  Boxes that
    // hold no key of the item come from a plane past the pool, which reads as
    // zeros and touches no memory.
    const int lw = warp - kLoadWarp0;
    const bool load_v = lw >= 2;                      // warps 8, 9: V ring
    const int nslots = load_v ? kVSlots : kKSlots;
    const int slot0 = load_v ? kKSlots : 0;           // the ring's first barrier / smem slot
    const int wl = lw & 1;                            // this warp fills the ring slots s with s % 2 == wl
    const uint32_t q_bytes = C::KATOMS * p.q_rows * 128;
    if (lane == 0) {
      if (lw == 0) prefetch_tmap(&tmap_q);
      prefetch_tmap(load_v ? &tmap_v : &tmap_k);
    }
    // Lane i holds the raw page-table entry of box i of an item (keys [16 i, 16 i + 16)
    // from the item's first tile; an item spans at most 4 tiles = 32 boxes); boxes that
    // hold no key of the item read no entry.  Read one item ahead and checked only where
    // it is used, so that the load's latency hides behind the current item.
    auto item_pages = [&](const DItem& it) -> int {
      int ph = 0;
      const int tok0 = it.j0 * kBT + lane * kBox;
      if (lane < it.nt * 8 && tok0 + kBox > it.t_begin && tok0 < it.t_end)
        ph = p.page_table[static_cast<size_t>(it.b) * p.max_pages + tok0 / p.page_size];
      return ph;
    };
    int T = 0, qn = 0;
    bool ok = true;
    int k = blockIdx.x;
    DItem cur = item_at(p, k, item_len(p, k));
    int ph_cur = item_pages(cur);
    int len_next = item_len(p, k + gridDim.x);
    for (int r = 0; r < n_rounds && ok; ++r, k += gridDim.x) {
      // next item's pages and the item after's length: loads in flight during this item
      const int len_after = item_len(p, k + 2 * gridDim.x);
      const DItem nxt = item_at(p, k + gridDim.x, len_next);
      const int ph_nxt = item_pages(nxt);
      const DItem it = cur;
      const int ph_it = ph_cur;
      cur = nxt;
      ph_cur = ph_nxt;
      len_next = len_after;
      if (it.nt == 0) continue;
      if (lw == 0 && lane == 0) {
        const int qb = qn & 1;
        if (qn >= 2) ok = mbar_wait(&q_empty[qb], ((qn >> 1) - 1) & 1, abort_flag, p.err);
        if (ok) {
          mbar_arrive_expect_tx(&q_full[qb], q_bytes);
          for (int a = 0; a < C::KATOMS; ++a)
            tma_load_3d(sQ + qb * C::Q_BYTES + a * C::Q_ATOM, &tmap_q, &q_full[qb], a * 64, it.g * G, it.b);
        }
      }
      if (lw == 0) ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ++qn;
      for (int jj = 0; jj < it.nt && ok; ++jj) {
        const int t = T + jj;                        // the ring's load t
        const int rs = t % nslots;
        if (rs % 2 != wl) continue;
        const int st = slot0 + rs;
        // lane rb + 8 a copies box rb (keys [16 rb, 16 rb + 16) of the tile) of atom a
        const int rb = lane & 7, a = lane >> 3;
        int ph = __shfl_sync(0xffffffffu, ph_it, (jj * 8 + rb) & 31);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], ((t / nslots) & 1) ^ 1, abort_flag, p.err))))
          break;
        uint64_t* bar = FP8 ? &raw_full[st] : &full[st];
        if (lane == 0) mbar_arrive_expect_tx(bar, FP8 ? kBT * D : C::TILE_BYTES);
        __syncwarp();   // the barrier is armed before any box can land
        if (lane < (FP8 ? 8 : 8 * C::KATOMS)) {
          const int tok0 = (it.j0 + jj) * kBT + rb * kBox;
          if (!(tok0 + kBox > it.t_begin && tok0 < it.t_end)) {
            ph = p.num_pages;   // no key of the item: a plane past the pool, read as zeros
          } else if (ph < 0 || ph >= p.num_pages) {   // never read outside the pool
            record_error(p.err, ATTN_ERRBIT_BADPAGE);
            ph = 0;
          }
          if constexpr (FP8)   // one box per page of the head: 16 rows x D codes, row-major
            tma_load_3d(sRing + st * C::TILE_BYTES + RAW_OFF + rb * kBox * D, load_v ? &tmap_v : &tmap_k, bar, 0,
                        tok0 % p.page_size, ph * p.Hkv + it.g);
          else
            tma_load_3d(sRing + st * C::TILE_BYTES + a * C::ATOM_BYTES + rb * kBox * 128,
                        load_v ? &tmap_v : &tmap_k, bar, a * 64, tok0 % p.page_size, ph * p.Hkv + it.g);
        }
      }
      T += it.nt;
    }
    // this warp's last copies must land before the CTA may exit (normally consumed already)
    for (int t = T - 1; t >= 0 && t >= T - nslots; --t)
      if ((t % nslots) % 2 == wl)
        mbar_wait(FP8 ? &raw_full[slot0 + t % nslots] : &full[slot0 + t % nslots], (t / nslots) & 1, nullptr,
                  p.err);
    if (lw == 0 && lane == 0)
      for (int m = max(0, qn - 2); m < qn; ++m) mbar_wait(&q_full[m & 1], (m >> 1) & 1, nullptr, p.err);
  } else if (FP8 && warp >= kConvWarp0) {
    // ------------------------------------------------------------ converter warps 10-13 (FP8)
    // Warps 10, 11 rewrite the K tiles t with t % kKSlots % 2 = 0, 1, warps 12,
    // 13 the V tiles likewise: each slot has one converter, which takes that
    // slot's tiles in order.  A slot's D-byte rows of codes sit row-major in its
    // upper half; the converter turns them into f16 in the 128-byte-swizzled
    // layout of a 16-bit tile, in place.  Rows go in increasing order, 32 or 64
    // at a time, each batch read completely before any of it is written: the
    // f16 row r lands on code rows of its own batch or earlier ones, never on a
    // code row still to be read.  Warp 10 also rewrites each
    // item's queries (bf16, landed by TMA) as f16 in place.
    const int cw = warp - kConvWarp0;
    const bool conv_v = cw >= 2;
    const int nslots = conv_v ? kVSlots : kKSlots;
    const int slot0 = conv_v ? kKSlots : 0;
    const int wl = cw & 1;
    constexpr int LPR = D / 16;                       // lanes per row: 16 codes (one 16-byte load) each
    constexpr int RPS = 32 / LPR;                     // rows per step
    const int lr = lane / LPR, c = lane % LPR;        // row within the step, 16-code chunk of the row
    int T = 0, qn = 0;
    bool ok = true;
    int len_cur = item_len(p, blockIdx.x);
    for (int r = 0; r < n_rounds && ok; ++r) {
      const int k = blockIdx.x + r * gridDim.x;
      const int len_next = item_len(p, k + gridDim.x);
      const DItem it = item_at(p, k, len_cur);
      len_cur = len_next;
      if (it.nt == 0) continue;
      if (cw == 0) {   // the item's queries: bf16 -> f16, in place
        const int qb = qn & 1;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&q_full[qb], (qn >> 1) & 1, abort_flag, p.err)))) break;
        uint4* qv = reinterpret_cast<uint4*>(sQ + qb * C::Q_BYTES);
        for (int i = lane; i < C::Q_BYTES / 16; i += 32) {   // every row (rows past q_rows feed ignored columns)
          uint4 u = qv[i];
          uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2 h = __floats2half2_rn(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
            w[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          qv[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&q_conv[qb]);
      }
      ++qn;
      for (int jj = 0; jj < it.nt && ok; ++jj) {
        const int t = T + jj;
        const int rs = t % nslots;
        if (rs % 2 != wl) continue;
        const int st = slot0 + rs;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&raw_full[st], (t / nslots) & 1, abort_flag, p.err)))) break;
        uint8_t* slot = sRing + st * C::TILE_BYTES;
        const uint4* raw = reinterpret_cast<const uint4*>(slot + RAW_OFF);
        constexpr int BATCH = 8;                      // steps whose codes are read before any is written
        for (int r0 = 0; r0 < kBT; r0 += RPS * BATCH) {
          uint4 u[BATCH];
#pragma unroll
          for (int b = 0; b < BATCH; ++b) u[b] = raw[(r0 + b * RPS + lr) * LPR + c];
          __syncwarp();   // the batch's code rows are read before any of its f16 rows is written
#pragma unroll
          for (int b = 0; b < BATCH; ++b) {
            const int row = r0 + b * RPS + lr;
            const uint32_t w[4] = {u[b].x, u[b].y, u[b].z, u[b].w};
            uint32_t h[8];   // 16 f16: elements 16 c .. 16 c + 15 of the row
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const unsigned short lo = static_cast<unsigned short>(w[e]), hi = static_cast<unsigned short>(w[e] >> 16);
              asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[2 * e]) : "h"(lo));
              asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[2 * e + 1]) : "h"(hi));
            }
            // two 16-byte chunks of atom (16 c) / 64, chunks 2 (c % 4) and 2 (c % 4) + 1 of the row, swizzled
            const int atom = c / 4, q0 = 2 * (c % 4);
            uint8_t* rowp = slot + atom * C::ATOM_BYTES + row * 128;
            *reinterpret_cast<uint4*>(rowp + ((q0 ^ (row & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(rowp + (((q0 + 1) ^ (row & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
          }
          __syncwarp();
        }
        fence_proxy_async_smem();   // the tensor cores read the tile through the async proxy
        mbar_arrive(&full[st]);
      }
      T += it.nt;
    }
  } else if (warp == kSWarp || warp == kPvWarp) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads issue the products, so that the issue cost of one (tens of
    // cycles per instruction, whatever its size) does not delay the other:
    // warp 4 the scores S^T(t) = K_t Q^T, warp 5 the outputs O += P(t) V_t.
    // Tile t's K is load t of the K ring and its V load t of the V ring.
    if (lane == 0) {
      const bool is_s = (warp == kSWarp);
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kNH, 0, 0, FP8);   // FP8: f16 operands
      constexpr uint32_t idesc_pv = idesc_bf16_f32(64, D, 0, 1, FP8);
      constexpr uint32_t kHi = sw128_desc_hi(1024);   // 8-row groups 1024 B apart
      const uint32_t q_lo0 = sw128_desc_lo(smem_u32(sQ), 16);
      const uint32_t p_lo0 = sw128_desc_lo(smem_u32(sP), 16);
      const uint32_t k_lo0 = sw128_desc_lo(smem_u32(sRing), 16);
      const uint32_t v_lo0 = sw128_desc_lo(smem_u32(sRing), C::ATOM_BYTES);   // MN-major: atoms 16 KB apart
      int qn = 0, T = 0, ic = 0;
      bool ok = true;
      auto wait_load = [&](int t, int& st) -> bool {   // tile t of this issuer's ring has landed
        const int ns = is_s ? kKSlots : kVSlots;
        st = (is_s ? 0 : kKSlots) + t % ns;
        const bool r = mbar_wait(&full[st], (t / ns) & 1, abort_flag, p.err);
        tc_fence_after();
        return r;
      };
      // V rows of page boxes that straddle the item's key range [t_begin, t_end)
      // hold keys outside it (slots after the last token may hold anything):
      // zero them before P V reads them.  Whole boxes outside arrive as zeros.
      auto clear_v_rows = [&](int st, int tile0, const DItem& it) {
        const int lo = it.t_begin - tile0, hi = it.t_end - tile0;   // valid rows [lo, hi) of the tile
        int r0[2] = {0, 0}, r1[2] = {0, 0};
        if (lo > 0 && lo < kBT && (lo % kBox) != 0) {
          r0[0] = lo - lo % kBox;
          r1[0] = lo;
        }
        if (hi > 0 && hi < kBT && (hi % kBox) != 0) {
          r0[1] = hi;
          r1[1] = hi - hi % kBox + kBox;
        }
        if (r1[0] <= r0[0] && r1[1] <= r0[1]) return;
        for (int e = 0; e < 2; ++e)
          for (int a = 0; a < C::KATOMS; ++a) {
            const uint32_t base = smem_u32(sRing + st * C::TILE_BYTES + a * C::ATOM_BYTES);
            for (int rr = r0[e]; rr < r1[e]; ++rr)   // a 128-byte row holds one key under the swizzle
              for (int c = 0; c < 128; c += 16)
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(base + rr * 128 + c), "r"(0u)
                             : "memory");
          }
        fence_proxy_async_smem();
      };
      int len_cur = item_len(p, blockIdx.x);
      for (int r = 0; r < n_rounds && ok; ++r) {
        const int k = blockIdx.x + r * gridDim.x;
        const int len_next = item_len(p, k + gridDim.x);   // in flight during this item
        const DItem it = item_at(p, k, len_cur);
        len_cur = len_next;
        if (it.nt == 0) continue;
        if (is_s) {
          const int qb = qn & 1;
          if (!(ok = mbar_wait(FP8 ? &q_conv[qb] : &q_full[qb], (qn >> 1) & 1, abort_flag, p.err))) break;
          tc_fence_after();
          for (int jj = 0; jj < it.nt && ok; ++jj) {
            const int t = T + jj, sb = t & 1;
            int st;
            if (!(ok = wait_load(t, st))) break;
            if (t >= 2) {   // the softmax has loaded S^T(t - 2)
              if (!(ok = mbar_wait(&s_free[sb], ((t >> 1) - 1) & 1, abort_flag, p.err))) break;
              tc_fence_after();
            }
            const uint32_t a_lo = k_lo0 + ((st * C::TILE_BYTES) >> 4);
            const uint32_t b_lo = q_lo0 + ((qb * C::Q_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t ka = ((kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32) >> 4;
              const uint32_t kb = ((kk >> 2) * C::Q_ATOM + (kk & 3) * 32) >> 4;
              mma_ss(tmem + C::S_COL + kNH * sb, desc64(a_lo + ka, kHi), desc64(b_lo + kb, kHi), idesc_s,
                     kk > 0 ? 1u : 0u);
            }
            mma_commit(&s_ready[sb]);
            mma_commit(&empty[st]);
            if (jj == it.nt - 1) mma_commit(&q_empty[qb]);
          }
          ++qn;
        } else {
          const int ob = ic & 1;
          for (int jj = 0; jj < it.nt && ok; ++jj) {
            const int t = T + jj, pb = t & 1;
            int st;
            if (!(ok = wait_load(t, st))) break;
            clear_v_rows(st, (it.j0 + jj) * kBT, it);
            if (!(ok = mbar_wait(&p_ready[pb], (t >> 1) & 1, abort_flag, p.err))) break;
            tc_fence_after();
            if (jj == 0 && ic >= 2) {   // item ic - 2 has read O buffer ob out
              if (!(ok = mbar_wait(&o_free[ob], ((ic >> 1) - 1) & 1, abort_flag, p.err))) break;
              tc_fence_after();
            }
            const uint32_t a_lo = p_lo0 + ((pb * C::P_BYTES) >> 4);
            const uint32_t b_lo = v_lo0 + ((st * C::TILE_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < kBT / 16; ++kk) {
              const uint32_t ka = ((kk >> 2) * C::P_ATOM + (kk & 3) * 32) >> 4;
              const uint32_t kb = (kk * 16 * 128) >> 4;
              mma_ss(tmem + C::O_COL + D * ob, desc64(a_lo + ka, kHi), desc64(b_lo + kb, kHi), idesc_pv,
                     (kk > 0 || jj > 0) ? 1u : 0u);
            }
            mma_commit(&p_free[pb]);
            mma_commit(&empty[st]);
            if (jj == it.nt - 1) mma_commit(&o_full[ob]);
          }
          ++ic;
        }
        T += it.nt;
      }
      // everything this thread issued must be complete before tensor memory is released
      mma_commit(&drain[is_s ? 0 : 1]);
      mbar_wait(&drain[is_s ? 0 : 1], 0, nullptr, p.err);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int rl = threadIdx.x;                        // key within the tile, TMEM lane of S^T
    const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
    int T = 0, ic = 0;
    // ok: this warp's status.  A warp whose wait gave up does no more work but
    // still reaches the next named barrier, where the four warps exchange their
    // status and leave together (quit), so that no warp waits there alone.
    bool ok = true, quit = false;
    float m_ref[G], l_part[G];
    int len_cur = item_len(p, blockIdx.x);
    for (int r = 0; r < n_rounds && !quit; ++r) {
      const int k = blockIdx.x + r * gridDim.x;
      const int len_next = item_len(p, k + gridDim.x);   // in flight during this item
      const DItem it = item_at(p, k, len_cur);
      if (rl == 0 && k < p.n_items && it.s == 0 && it.g == 0 &&
          len_cur > min(p.max_seq_len, p.max_pages * p.page_size))
        record_error(p.err, ATTN_ERRBIT_BADPAGE);   // longer than the table or max_seq_len: truncated
      len_cur = len_next;
      if (it.nt == 0) continue;
      const int ob = ic & 1;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_ref[h] = -INFINITY;
        l_part[h] = 0.f;
      }
      for (int jj = 0; jj < it.nt; ++jj) {
        const int t = T + jj, sb = t & 1;
        float s[kNH];
        bool wok = ok && mbar_wait(&s_ready[sb], (t >> 1) & 1, abort_flag, p.err);
        wok = __all_sync(0xffffffffu, wok);
        if (wok) {
          tc_fence_after();
          tmem_ld16f(tmem + lane_bits + C::S_COL + kNH * sb, s);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&s_free[sb]);
        }
        const int key = (it.j0 + jj) * kBT + rl;
        const bool vis = wok && key >= it.t_begin && key < it.t_end;
        float x[G];
        float* rd = red + (t & 1) * 4 * kNH;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          x[h] = vis ? s[h] * p.scale_log2 : -INFINITY;
          float mx = x[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (lane == 0) rd[warp * kNH + h] = mx;
        }
        if (lane == 0) okv[(t & 1) * 4 + warp] = wok ? 1 : 0;
        named_barrier_sync(1, 128);
        if (!(okv[(t & 1) * 4 + 0] && okv[(t & 1) * 4 + 1] && okv[(t & 1) * 4 + 2] && okv[(t & 1) * 4 + 3])) {
          quit = true;   // every warp leaves together
          break;
        }
        bool resc = false;
        float alpha[G], pr[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mt = fmaxf(fmaxf(rd[h], rd[kNH + h]), fmaxf(rd[2 * kNH + h], rd[3 * kNH + h]));
          alpha[h] = 1.f;
          if (mt > m_ref[h] + kTau) {
            alpha[h] = (m_ref[h] == -INFINITY) ? 0.f : ex2(m_ref[h] - mt);
            resc |= (m_ref[h] != -INFINITY);
            l_part[h] *= alpha[h];
            m_ref[h] = mt;
          }
          pr[h] = ex2(x[h] - m_ref[h]);   // exactly 0 for keys outside the item
          l_part[h] += pr[h];
        }
        // P buffer t % 2 is free once P(t - 2) V is complete; O holds P(t - 1) V once that is complete
        bool wok2 = true;
        if (t >= 2) wok2 = mbar_wait(&p_free[sb], ((t >> 1) - 1) & 1, abort_flag, p.err);
        if (resc && jj > 0 && wok2) wok2 = mbar_wait(&p_free[sb ^ 1], ((t - 1) >> 1) & 1, abort_flag, p.err);
        wok2 = __all_sync(0xffffffffu, wok2);
        if (!wok2) {
          ok = false;   // stops at the next barrier (tile or read-out), together with the other warps
          continue;
        }
        tc_fence_after();
        if (resc && jj > 0 && warp == 0) {   // O row h *= alpha[h] (rows are heads, TMEM lanes 0..31)
          float a = 1.f;
#pragma unroll
          for (int h = 0; h < G; ++h) a = (lane == h) ? alpha[h] : a;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + C::O_COL + D * ob + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
            tmem_st32(tmem + C::O_COL + D * ob + 32 * c, o);
          }
          tmem_wait_st();
        }
        // column rl of P: row h, 64-key atom rl / 64, 16-byte chunk (rl % 64) / 8 swizzled by row
        const uint32_t pbase = smem_u32(sP) + sb * C::P_BYTES + (rl >> 6) * C::P_ATOM + (rl & 7) * 2;
        const int chunk = (rl & 63) >> 3;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          unsigned short v;
          if constexpr (FP8) {
            const __half hv = __float2half_rn(pr[h]);
            v = *reinterpret_cast<const unsigned short*>(&hv);
          } else {
            const __nv_bfloat16 bv = __float2bfloat16_rn(pr[h]);
            v = *reinterpret_cast<const unsigned short*>(&bv);
          }
          const uint32_t addr = pbase + h * 128 + ((chunk ^ (h & 7)) << 4);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
        }
        fence_proxy_async_smem();   // the MMA reads P through the async proxy
        tc_fence_before();
        mbar_arrive(&p_ready[sb]);
      }
      if (quit) break;
      // ---- read-out: O row h / l_h -> the split's partial output, and its base-2 log-sum-exp
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float ls = l_part[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
        if (lane == 0) lred[warp * kNH + h] = ls;
      }
      bool wok = ok && mbar_wait(&o_full[ob], (ic >> 1) & 1, abort_flag, p.err);
      wok = __all_sync(0xffffffffu, wok);
      if (lane == 0) okv[8 + warp] = wok ? 1 : 0;
      named_barrier_sync(1, 128);
      if (!(okv[8] && okv[9] && okv[10] && okv[11])) {
        quit = true;
        break;
      }
      tc_fence_after();
      if (warp == 0) {
        float mr = m_ref[0];
#pragma unroll
        for (int h = 1; h < G; ++h) mr = (lane == h) ? m_ref[h] : mr;
        const float lsum = (lane < G) ? (lred[lane] + lred[kNH + lane]) + (lred[2 * kNH + lane] + lred[3 * kNH + lane])
                                      : 0.f;
        const float inv = (lsum > 0.f) ? 1.f / lsum : 0.f;
        const size_t row = (static_cast<size_t>(it.b) * p.Hq + it.g * G + lane) * p.max_splits + it.s;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + C::O_COL + D * ob + 32 * c, o);
          tmem_wait_ld();
          if (lane < G) {
            float4* dst = reinterpret_cast<float4*>(p.ws_o + row * D + 32 * c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                   __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
          }
        }
        if (lane < G) p.ws_lse[row] = (lsum > 0.f) ? mr + log2f(lsum) : -INFINITY;
      }
      tc_fence_before();
      mbar_arrive(&o_free[ob]);
      T += it.nt;
      ++ic;
    }
    // if a wait gave up, the remaining partials stay unwritten and the error word records it
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, int G, bool FP8>
cudaError_t launch_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const TcParams& p,
                     cudaStream_t stream) {
  using C = TcCfg<D>;
  auto kern = decode_tc_kernel<D, G, FP8>;
  constexpr int kMaxDevices = 64;
  static int ready[kMaxDevices] = {};   // the shared-memory limit is set once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE) != 1) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(C::SMEM));
    if (e != cudaSuccess) return e;
    __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
  }
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(p.n_items < sms ? p.n_items : sms);
  kern<<<grid, tc_threads<FP8>(), C::SMEM, stream>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tc_split(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                   const int32_t* seq_lens, int page_size, int N, int Hq, int Hkv, int D,
                                   int num_pages, int max_pages, int max_seq_len, float scale, int window,
                                   int split_tokens, int max_splits, float* ws_o, float* ws_lse, unsigned int* err,
                                   cudaStream_t stream, bool fp8, float k_scale) {
  const int G = Hq / Hkv;
  if (split_tokens % kBT != 0 || page_size % kBox != 0) return cudaErrorInvalidValue;
  TcParams p{};
  p.k_pool = k_pool;
  p.v_pool = v_pool;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.ws_o = ws_o;
  p.ws_lse = ws_lse;
  p.err = err;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.num_pages = num_pages;
  p.max_pages = max_pages;
  p.page_size = page_size;
  p.max_seq_len = max_seq_len;
  p.window = window;
  p.split_tokens = split_tokens;
  p.max_splits = max_splits;
  const long long items = static_cast<long long>(N) * Hkv * max_splits;
  if (items <= 0) return cudaSuccess;
  if (items > (1LL << 30)) return cudaErrorInvalidValue;
  p.n_items = static_cast<int>(items);
  p.q_rows = Hq < kNH ? Hq : kNH;
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  CUtensorMap mq, mk, mv;
  // bf16 pools: 64-column boxes in the 128-byte swizzle; 8-bit pools: whole D-byte rows, row-major
  const int eb = fp8 ? 1 : 2, box_inner = fp8 ? D : 64;
  if (!make_tensor_map_3d(&mq, q, 2, D, Hq, N, 64, p.q_rows) ||
      !make_tensor_map_3d(&mk, k_pool, eb, D, page_size, num_pages * Hkv, box_inner, kBox, !fp8) ||
      !make_tensor_map_3d(&mv, v_pool, eb, D, page_size, num_pages * Hkv, box_inner, kBox, !fp8))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaErrorInvalidValue;
#define ATTN_TC_CASE(DD, GG)                                                              \
  if (D == DD && G == GG)                                                                 \
    e = fp8 ? launch_d<DD, GG, true>(mq, mk, mv, p, stream) : launch_d<DD, GG, false>(mq, mk, mv, p, stream);
  ATTN_TC_CASE(128, 1) ATTN_TC_CASE(128, 2) ATTN_TC_CASE(128, 4) ATTN_TC_CASE(128, 8)
  ATTN_TC_CASE(64, 1) ATTN_TC_CASE(64, 2) ATTN_TC_CASE(64, 4) ATTN_TC_CASE(64, 8)
#undef ATTN_TC_CASE
  return e;
}

}  // namespace attn
