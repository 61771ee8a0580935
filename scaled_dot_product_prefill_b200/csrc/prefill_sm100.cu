// prefill_sm100.cu -- bf16 attention prefill on the fifth-generation tensor cores.
//
// What is computed: O = softmax(Q K^T * scale + mask) V per (batch, query
// head), with the causal / sliding-window masks and the GQA head map of the
// public header.  The n x n score matrix is never written to memory: keys
// are visited a tile at a time and an online softmax (running row maximum
// and sum; earlier partial results rescaled when the maximum grows) gives
// exactly the softmax of the full row ("Attention From Scratch" README,
// section "Flash Attention"; "Taking LLMs apart (2)", section
// "FlashAttention"; "Attention mechanism explained", section 7).
//
// How.  A work item is a block of 2 x 128 query rows of one (batch, head).
// The kernel is persistent: one CTA per SM walks the items in order of
// decreasing cost (later causal blocks first), dealt out in a snake so that
// the SMs finish together.  Each CTA has 12 warps:
//   warps 0-3  softmax group 0: thread t owns row t of query tile 0
//   warps 4-7  softmax group 1: the same for query tile 1
//   warp 8     TMA producer: Q of each item, then K_j / V_j tiles into a ring
//              of shared-memory slots (128-byte swizzle, no multicast); one
//              thread for dense K/V, the whole warp for page boxes
//   warp 9     MMA issuer (one thread) and tensor-memory owner
//   warps 10-11 idle (complete the third warpgroup for the register split)
// Tensor memory (512 columns x 128 lanes, fp32):
//   S_i = Q_i K_j^T   columns [128 i, 128 i + 128)      (A and B in smem)
//   P_i (bf16)        written over the first 64 columns of S_i by the softmax
//   O_i += P_i V_j    columns [256 + D i, 256 + D i + D) (A = P in tmem)
// The MMA thread alternates the two query tiles: as soon as group i hands
// back P_i(j) it issues P_i(j) V_j and then S_i(j+1), so one group's softmax
// overlaps the other group's matrix products.  Tensor-core work is in
// order, so the commit that signals S_i(j+1) also covers P_i(j) V_j: the
// softmax thread may then rescale O_i without another barrier.  The
// reference maximum only moves when a score exceeds it by 2^8 (in
// probability), so rescaling is rare after the first key tile and the
// result stays exact.  Key tiles that the mask hides from every row of a
// query tile are never loaded or multiplied; element masks are applied only
// on tiles that straddle a mask edge.
//
// At D = 64 tensor memory has room for P buffers of their own (Cfg::SEP_P):
// the softmax releases S_i as soon as it has loaded it, the MMA thread
// computes S_i(j+1) while the exponentials of tile j run, and each P_i V_j
// signals its own completion.  PAGED kernels read K/V through a page table
// as page-sized TMA boxes.
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <pthread.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int BM = 128;          // query rows per tile
constexpr int NQ = 2;            // query tiles per work item
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kTau = 8.0f;     // lazy-rescale threshold, log2 units

template <int D>
struct Cfg {
  static constexpr int BN = 128;                      // keys per tile
  // 12 warps (3 warpgroups) and a register split (setmaxnreg works per
  // warpgroup): the two softmax groups hold a 128-column score row each; the
  // producer group (TMA and MMA warps, two idle warps) gets the rest.
  // 128 * (2 * SOFTMAX_REGS + PRODUCER_REGS) must fit the launch allocation
  // (threads * registers per thread), which the host checks before the first
  // launch.
  static constexpr int THREADS = 384;
  static constexpr int SOFTMAX_REGS = 208;
  static constexpr int PRODUCER_REGS = 88;
  static constexpr int KATOMS = D / 64;               // 64-column (128-byte) swizzle atoms
  static constexpr int TILE_BYTES = BN * D * 2;       // one K or V tile
  static constexpr int Q_BYTES = BM * D * 2;          // one query tile
  static constexpr int QBUF = (D == 128) ? 1 : 2;     // query buffers (items in flight)
  static constexpr int STAGES = (D == 128) ? 4 : 6;   // ring slots; K and V tiles alternate
  // D = 64 leaves room in tensor memory for P buffers of their own (SEP_P):
  // S_i [128 i, +128), P_i [256 + 64 i, +64), O_i [384 + 64 i, +64).  The
  // softmax then releases S_i as soon as it has loaded it, S_i(j+1) is
  // computed while the softmax of tile j is still running, and O_i is
  // rescaled after the exponentials.  D = 128 has no room: P_i is written
  // over the first 64 columns of S_i, O_i [256 + 128 i, +128).
  static constexpr bool SEP_P = (D == 64);
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;                // + BN * i
  static constexpr uint32_t P_COL = SEP_P ? 256 : 0;  // + P_STRIDE * i
  static constexpr uint32_t P_STRIDE = SEP_P ? 64 : BN;
  static constexpr uint32_t O_COL = SEP_P ? 384 : NQ * BN;  // + D * i
  static constexpr size_t SMEM = 1024 /*align*/ + QBUF * NQ * Q_BYTES + STAGES * TILE_BYTES + 256;
};

struct Params {
  int B, Hq, Hkv, Sq, Skv, causal, window, n_qblocks, n_items;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;           // [B, Hq, Sq] natural-log log-sum-exp, or null
  unsigned int* err;
  // paged K/V (the PAGED kernels): K and V come from [num_pages, Hkv, page_size, D]
  // pools through page_table [B, max_pages]; sequence b has seq_lens[b] keys
  // (at most Skv, the caller's bound), and its Sq queries are the last Sq of them.
  const int32_t* page_table;
  const int32_t* seq_lens;
  int page_size, box_rows, max_pages, num_pages;
};

struct Item {
  int bh, b, g, q_row0, skv;   // skv: keys of this item's sequence
  int lo[NQ], hi[NQ];   // key-tile range per query tile (empty if hi <= lo)
  int lo_all, hi_all;   // union; empty if hi_all <= lo_all
};

// The r-th item of this CTA (snake over cost-ordered items), or -1.
__device__ __forceinline__ int item_index(const Params& p, int r) {
  const int P = gridDim.x, c = blockIdx.x;
  const int k = r * P + ((r & 1) ? (P - 1 - c) : c);
  return k < p.n_items ? k : -1;
}

template <int BN, bool PAGED>
__device__ __forceinline__ Item make_item(const Params& p, int k) {
  Item it;
  const int BH = p.B * p.Hq;
  it.bh = k % BH;
  const int qb = p.n_qblocks - 1 - k / BH;   // costliest (latest) query blocks first
  it.b = it.bh / p.Hq;
  it.g = (it.bh % p.Hq) / (p.Hq / p.Hkv);
  it.q_row0 = qb * (NQ * BM);
  it.skv = p.Skv;
  if constexpr (PAGED) {
    const int L = p.seq_lens[it.b];
    const int cap = min(p.Skv, p.max_pages * p.page_size);
    if (L > cap) record_error(p.err, ATTN_ERRBIT_BADPAGE);
    it.skv = max(0, min(L, cap));
  }
  const int off = it.skv - p.Sq;
  const int n_kt = (it.skv + BN - 1) / BN;
  it.lo_all = 1 << 30;
  it.hi_all = 0;
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    const int r0 = it.q_row0 + BM * i;
    const int r1 = min(r0 + BM, p.Sq);   // exclusive
    int lo = 0, hi = 0;
    if (r0 < p.Sq) {
      if (!p.causal) {
        hi = n_kt;
      } else {
        const int last_key = min(r1 - 1 + off, it.skv - 1);
        const int first_key = (p.window > 0) ? max(0, r0 + off - p.window + 1) : 0;
        if (last_key >= first_key && last_key >= 0) {
          lo = first_key / BN;
          hi = last_key / BN + 1;
        }
      }
    }
    it.lo[i] = lo;
    it.hi[i] = hi;
    if (hi > lo) {
      it.lo_all = min(it.lo_all, lo);
      it.hi_all = max(it.hi_all, hi);
    }
  }
  if (it.hi_all <= 0) it.lo_all = it.hi_all = 0;
  return it;
}

__device__ __forceinline__ bool active(const Item& it, int i, int j) { return j >= it.lo[i] && j < it.hi[i]; }

// True if every (row, key) pair of query rows [r0, r0+BM) x key tile j is visible
// (skv keys in the sequence).
template <int BN>
__device__ __forceinline__ bool tile_unmasked(const Params& p, int skv, int r0, int j) {
  const int off = skv - p.Sq;
  const int k0 = j * BN, k1 = j * BN + BN - 1;
  if (k1 >= skv) return false;
  if (!p.causal) return true;
  if (k1 > r0 + off) return false;
  if (p.window > 0 && k0 <= r0 + BM - 1 + off - p.window) return false;
  return true;
}

// PAGED selects K/V through a page table (chunked prefill over a paged cache)
// instead of dense [B, Hkv, Skv, D] tensors; the dense kernel carries none of
// the paged code.
template <int D, bool PAGED>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using C = Cfg<D>;
  constexpr int BN = C::BN;
  constexpr int STAGES = C::STAGES, QBUF = C::QBUF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                                   // [QBUF][NQ][KATOMS][BM rows x 128 B]
  uint8_t* sRing = smem + QBUF * NQ * C::Q_BYTES;       // [STAGES][KATOMS][BN rows x 128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRing + STAGES * C::TILE_BYTES);
  uint64_t* q_full = bars;                              // QBUF
  uint64_t* q_empty = q_full + QBUF;                    // QBUF
  uint64_t* full = q_empty + QBUF;                      // STAGES
  uint64_t* empty = full + STAGES;                      // STAGES
  uint64_t* s_ready = empty + STAGES;                   // NQ
  uint64_t* p_ready = s_ready + NQ;                     // NQ
  uint64_t* o_done = p_ready + NQ;                      // NQ: O_i final (SEP_P: each P_i V done)
  uint64_t* s_free = o_done + NQ;                       // NQ: S_i loaded by the softmax (SEP_P)
  uint64_t* drain = s_free + NQ;                        // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rounds = (p.n_items + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int q = 0; q < QBUF; ++q) {
      mbar_init(&q_full[q], 1);
      mbar_init(&q_empty[q], 1);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&s_ready[i], 1);
      mbar_init(&p_ready[i], 4 * 32);
      mbar_init(&o_done[i], 1);
      mbar_init(&s_free[i], 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up above overlaps the tail of the kernel before; global memory only from here on
  grid_dependency_wait();

  if (warp >= 8) {
   // ------------------------------------------------------------ producer warpgroup
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::PRODUCER_REGS));
   if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    // Dense: one thread.  Paged: the whole warp, so that the page-table
    // entries of a tile are read by one load and its page boxes issued by
    // one instruction (lane 0 still arms the barriers and loads Q).
    if (PAGED || lane == 0) {
      const bool lead = (lane == 0);
      auto uni = [&](bool v) -> bool {   // one outcome for the whole warp
        if constexpr (PAGED) return __all_sync(0xffffffffu, v);
        return v;
      };
      if (lead) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
      }
      int n = 0, qn = 0;
      bool ok = true;
      for (int r = 0; r < n_rounds && ok; ++r) {
        const int k = item_index(p, r);
        if (k < 0) continue;
        const Item it = make_item<BN, PAGED>(p, k);
        if (it.hi_all <= it.lo_all) continue;
        const int qb = qn % QBUF;
        if (qn >= QBUF && !(ok = uni(mbar_wait(&q_empty[qb], ((qn / QBUF) - 1) & 1, abort_flag, p.err)))) break;
        if (lead) {
          mbar_arrive_expect_tx(&q_full[qb], NQ * C::Q_BYTES);
          for (int i = 0; i < NQ; ++i)
            for (int a = 0; a < C::KATOMS; ++a)
              tma_load_3d(sQ + ((qb * NQ + i) * C::KATOMS + a) * BM * 128, &tmap_q, &q_full[qb], a * 64,
                          it.q_row0 + BM * i, it.bh);
        }
        ++qn;
        const int kv_plane = it.b * p.Hkv + it.g;
        // PAGED: the physical page of this lane's box of key tile j (lane rb + nb * a
        // copies box rb of swizzle atom a), or the pool size for a box past the end
        // of the sequence.  K_j and V_j share it, and it is read one tile ahead, so
        // that the page-table load overlaps the wait for a free ring slot.
        auto page_of = [&](int j) -> int {
          if constexpr (!PAGED) {
            return 0;
          } else {
            const int nb = BN / p.box_rows;
            int ph = p.num_pages;                 // plane ph * Hkv + g is past the pool's planes
            if (lane < nb * C::KATOMS) {
              const int key0 = j * BN + (lane % nb) * p.box_rows;
              if (key0 < it.skv) {
                ph = p.page_table[static_cast<size_t>(it.b) * p.max_pages + key0 / p.page_size];
                if (ph < 0 || ph >= p.num_pages) {  // never read outside the pool
                  record_error(p.err, ATTN_ERRBIT_BADPAGE);
                  ph = 0;
                }
              }
            }
            return ph;
          }
        };
        auto load = [&](bool is_v, int j, int ph) -> bool {   // next ring slot <- K_j or V_j
          const int st = n % STAGES;
          if (!uni(mbar_wait(&empty[st], ((n / STAGES) & 1) ^ 1, abort_flag, p.err))) return false;
          if (lead) mbar_arrive_expect_tx(&full[st], C::TILE_BYTES);
          const CUtensorMap* tm = is_v ? &tmap_v : &tmap_k;
          if constexpr (!PAGED) {
            for (int a = 0; a < C::KATOMS; ++a)
              tma_load_3d(sRing + st * C::TILE_BYTES + a * BN * 128, tm, &full[st], a * 64, j * BN, kv_plane);
          } else {
            // the key tile is assembled from page boxes of box_rows rows each; a
            // box lands at its row offset inside the swizzled tile, so the MMA
            // sees the same layout as a dense load
            // boxes that start past the sequence end read no page: their plane
            // coordinate is past the pool, so the copy fills them with zeros.
            // Lane rb + nb * a copies box rb of swizzle atom a (at most 8 x 2).
            __syncwarp();   // the barrier is armed before any box can land
            const int nb = BN / p.box_rows;
            if (lane < nb * C::KATOMS) {
              const int rb = lane % nb, a = lane / nb;
              const int key0 = j * BN + rb * p.box_rows;
              tma_load_3d(sRing + st * C::TILE_BYTES + a * BN * 128 + rb * p.box_rows * 128, tm, &full[st],
                          a * 64, key0 % p.page_size, ph * p.Hkv + it.g);
            }
          }
          ++n;
          return true;
        };
        // load order = the MMA thread's consumption order
        if constexpr (C::SEP_P) {   // K_lo, then K_{j+1} ahead of V_j
          int ph_j = page_of(it.lo_all);
          int ph_j1 = (it.lo_all + 1 < it.hi_all) ? page_of(it.lo_all + 1) : 0;
          ok = load(false, it.lo_all, ph_j);
          for (int j = it.lo_all; j < it.hi_all && ok; ++j) {
            const int ph_j2 = (j + 2 < it.hi_all) ? page_of(j + 2) : 0;
            if (j + 1 < it.hi_all) ok = load(false, j + 1, ph_j1);
            if (ok) ok = load(true, j, ph_j);
            ph_j = ph_j1;
            ph_j1 = ph_j2;
          }
        } else {                    // K_j, V_j
          int ph_j = page_of(it.lo_all);
          for (int j = it.lo_all; j < it.hi_all && ok; ++j) {
            const int ph_j1 = (j + 1 < it.hi_all) ? page_of(j + 1) : 0;
            ok = load(false, j, ph_j);
            if (ok) ok = load(true, j, ph_j);
            ph_j = ph_j1;
          }
        }
      }
      // the last loads issued must land before the CTA may exit (normally already consumed)
      for (int k = max(0, n - STAGES); k < n; ++k) mbar_wait(&full[k % STAGES], (k / STAGES) & 1, nullptr, p.err);
    }
   } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
      constexpr uint32_t kHi = sw128_desc_hi(1024);   // 8-row groups 1024 B apart
      // descriptor low words at K step 0: Q tiles (K-major), ring slots as K (K-major)
      // and as V (MN-major, 64-column blocks BN*128 bytes apart); a K step adds a
      // compile-time offset in 16-byte units
      const uint32_t q_lo0 = sw128_desc_lo(smem_u32(sQ), 16);
      const uint32_t k_lo0 = sw128_desc_lo(smem_u32(sRing), 16);
      const uint32_t v_lo0 = sw128_desc_lo(smem_u32(sRing), BN * 128);
      int n = 0, qn = 0;
      int ts[NQ] = {0, 0};
      bool ok = true;

      auto issue_s = [&](int i, int qb, int st) {  // S_i = Q_i K^T from ring slot st
        const uint32_t d_tmem = tmem + C::S_COL + BN * i;
        const uint32_t a_lo = q_lo0 + (((qb * NQ + i) * C::Q_BYTES) >> 4);
        const uint32_t b_lo = k_lo0 + ((st * C::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = ((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4;
          mma_ss(d_tmem, desc64(a_lo + koff, kHi), desc64(b_lo + koff, kHi), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_ready[i]);
      };
      // Paged K/V: the page box that holds a sequence's last key also brings the
      // slots after it, whose contents are arbitrary.  Their scores are masked
      // and P is 0 there, but 0 * NaN is NaN, so the V rows past the end are
      // zeroed in shared memory before P.V reads them.  Boxes wholly past the
      // end arrive as zeros already.
      auto clear_v_tail = [&](int st, int j, int skv) {
        if constexpr (!PAGED) return;
        const int from = skv - j * BN;
        if (from <= 0 || from >= BN) return;
        const int to = min(BN, (from + p.box_rows - 1) / p.box_rows * p.box_rows);
        if (to <= from) return;
        for (int a = 0; a < C::KATOMS; ++a) {
          const uint32_t base = smem_u32(sRing + st * C::TILE_BYTES + a * BN * 128);
          for (int r = from; r < to; ++r)   // a 128-byte row holds the same key under the swizzle
            for (int c = 0; c < 128; c += 16)
              asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(base + r * 128 + c), "r"(0u)
                           : "memory");
        }
        fence_proxy_async_smem();
      };
      auto wait_slot = [&](int& st) -> bool {   // next ring slot, in load order
        st = n % STAGES;
        const bool r = mbar_wait(&full[st], (n / STAGES) & 1, abort_flag, p.err);
        ++n;
        tc_fence_after();
        return r;
      };

      if constexpr (C::SEP_P) {
        // Order per key tile j: S_i(j+1) as soon as softmax group i has loaded
        // S_i(j) (s_free), then P_i(j) V_j as soon as it has written P_i(j).
        int tf[NQ] = {0, 0};    // s_free phases consumed per tile
        for (int r = 0; r < n_rounds && ok; ++r) {
          const int k = item_index(p, r);
          if (k < 0) continue;
          const Item it = make_item<BN, PAGED>(p, k);
          if (it.hi_all <= it.lo_all) continue;
          const int qb = qn % QBUF;
          if (!(ok = mbar_wait(&q_full[qb], (qn / QBUF) & 1, abort_flag, p.err))) break;
          tc_fence_after();
          ++qn;
          int stK;
          if (!(ok = wait_slot(stK))) break;
#pragma unroll
          for (int i = 0; i < NQ; ++i)
            if (active(it, i, it.lo_all)) issue_s(i, qb, stK);
          mma_commit(&empty[stK]);
          if (it.hi_all - it.lo_all == 1) mma_commit(&q_empty[qb]);

          for (int j = it.lo_all; j < it.hi_all && ok; ++j) {
            if (j + 1 < it.hi_all) {
              int stK1;
              if (!(ok = wait_slot(stK1))) break;
#pragma unroll
              for (int i = 0; i < NQ; ++i) {
                if (!active(it, i, j + 1)) continue;
                if (active(it, i, j)) {   // S_i still holds tile j until the softmax has loaded it
                  if (!(ok = mbar_wait(&s_free[i], tf[i] & 1, abort_flag, p.err))) break;
                  tc_fence_after();
                  ++tf[i];
                }
                issue_s(i, qb, stK1);
              }
              if (!ok) break;
              mma_commit(&empty[stK1]);
              if (j + 1 == it.hi_all - 1) mma_commit(&q_empty[qb]);
            }
            int stV;
            if (!(ok = wait_slot(stV))) break;
            clear_v_tail(stV, j, it.skv);
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
              if (!active(it, i, j)) continue;
              if (!(ok = mbar_wait(&p_ready[i], ts[i] & 1, abort_flag, p.err))) break;
              tc_fence_after();
              ++ts[i];
              const uint32_t o_tmem = tmem + C::O_COL + D * i;
              const uint32_t vb_lo = v_lo0 + ((stV * C::TILE_BYTES) >> 4);
              const uint32_t acc0 = (j > it.lo[i]) ? 1u : 0u;
              const uint32_t p_tmem = tmem + C::P_COL + C::P_STRIDE * i;
#pragma unroll
              for (int kk = 0; kk < BN / 16; ++kk)
                mma_ts(o_tmem, p_tmem + kk * 8, desc64(vb_lo + ((kk * 16 * 128) >> 4), kHi), idesc_pv,
                       kk > 0 ? 1u : acc0);
              mma_commit(&o_done[i]);   // P_i free again, O_i current
            }
            if (!ok) break;
            mma_commit(&empty[stV]);
          }
          // tiles whose last S tile was loaded but never freed by a following S: consume the phase
#pragma unroll
          for (int i = 0; i < NQ; ++i) {
            if (it.hi[i] > it.lo[i] && ok) {
              if (!(ok = mbar_wait(&s_free[i], tf[i] & 1, abort_flag, p.err))) break;
              ++tf[i];
            }
          }
        }
      } else {
      for (int r = 0; r < n_rounds && ok; ++r) {
          const int k = item_index(p, r);
          if (k < 0) continue;
          const Item it = make_item<BN, PAGED>(p, k);
          if (it.hi_all <= it.lo_all) continue;
          const int qb = qn % QBUF;
          if (!(ok = mbar_wait(&q_full[qb], (qn / QBUF) & 1, abort_flag, p.err))) break;
          tc_fence_after();
          ++qn;
          // prologue: S_i(lo) for the tiles that start at the first key tile
          int stK;
          if (!(ok = wait_slot(stK))) break;
#pragma unroll
          for (int i = 0; i < NQ; ++i)
            if (active(it, i, it.lo_all)) issue_s(i, qb, stK);
          mma_commit(&empty[stK]);
          if (it.hi_all - it.lo_all == 1) mma_commit(&q_empty[qb]);

          for (int j = it.lo_all; j < it.hi_all && ok; ++j) {
            int stV;
            if (!(ok = wait_slot(stV))) break;
            clear_v_tail(stV, j, it.skv);
            const bool next = j + 1 < it.hi_all;
            int stK1 = -1;
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
              if (active(it, i, j)) {
                if (!(ok = mbar_wait(&p_ready[i], ts[i] & 1, abort_flag, p.err))) break;
                tc_fence_after();
                ++ts[i];
                const uint32_t o_tmem = tmem + C::O_COL + D * i;
                const uint32_t p_tmem = tmem + C::P_COL + C::P_STRIDE * i;
                const uint32_t vb_lo = v_lo0 + ((stV * C::TILE_BYTES) >> 4);
                const uint32_t acc0 = (j > it.lo[i]) ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                  mma_ts(o_tmem, p_tmem + kk * 8, desc64(vb_lo + ((kk * 16 * 128) >> 4), kHi), idesc_pv,
                         kk > 0 ? 1u : acc0);
                if (j == it.hi[i] - 1) mma_commit(&o_done[i]);
              }
              if (next && active(it, i, j + 1)) {
                if (stK1 < 0 && !(ok = wait_slot(stK1))) break;
                issue_s(i, qb, stK1);
              }
            }
            if (!ok) break;
            if (next && stK1 < 0 && !(ok = wait_slot(stK1))) break;   // K tile that no query tile needs
            mma_commit(&empty[stV]);
            if (next) mma_commit(&empty[stK1]);
            if (j == it.hi_all - 2) mma_commit(&q_empty[qb]);
          }
        }
      }
      // everything issued above must be complete before tensor memory is released
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err);
    }
   }
  } else {
    // ------------------------------------------------------------ softmax groups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFTMAX_REGS));
    const int i = warp >> 2;                 // query tile
    const int wq = warp & 3;                 // lane quarter of tensor memory
    const int rl = wq * 32 + lane;           // row within the tile
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_tmem = tmem + lane_bits + C::S_COL + BN * i;
    const uint32_t p_tmem = tmem + lane_bits + C::P_COL + C::P_STRIDE * i;
    const uint32_t o_tmem = tmem + lane_bits + C::O_COL + D * i;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    int t = 0, oc = 0;
    int pv = 0;   // SEP_P: P_i V products of this tile completed and waited for
    // O_i *= alpha (every row of the warp takes part when any row needs it)
    auto rescale_o = [&](bool later_tile, float alpha) {
      if (!__any_sync(0xffffffffu, later_tile && alpha != 1.f)) return;
      const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(o_tmem + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float x0, x1;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), x0, x1);
          o[e] = __float_as_uint(x0);
          o[e + 1] = __float_as_uint(x1);
        }
        tmem_st32(o_tmem + 32 * c, o);
      }
    };
    bool ok = true;

    for (int rr = 0; rr < n_rounds && ok; ++rr) {
      const int k = item_index(p, rr);
      if (k < 0) continue;
      const Item it = make_item<BN, PAGED>(p, k);
      const int my_lo = (i == 0) ? it.lo[0] : it.lo[1];
      const int my_hi = (i == 0) ? it.hi[0] : it.hi[1];
      const int r0 = it.q_row0 + BM * i;
      const int r = r0 + rl;                 // query row of this thread
      const bool store = r < p.Sq;
      __nv_bfloat16* orow = p.out + (static_cast<size_t>(it.bh) * p.Sq + r) * D;
      if (my_hi <= my_lo) {                  // no visible key for any row of this tile
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow);
          for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
          if (p.lse != nullptr) p.lse[static_cast<size_t>(it.bh) * p.Sq + r] = -INFINITY;
        }
        continue;
      }
      // visible keys of this row: [key_lo, key_hi]
      const int skv = it.skv;
      const int off = skv - p.Sq;
      const int key_hi = p.causal ? min(r + off, skv - 1) : skv - 1;
      const int key_lo = (p.causal && p.window > 0) ? r + off - p.window + 1 : 0;
      float m_ref = -INFINITY, l = 0.f;

      for (int j = my_lo; j < my_hi; ++j, ++t) {
        ok = mbar_wait(&s_ready[i], t & 1, abort_flag, p.err);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32f(s_tmem + 32 * c, s + 32 * c);
        tmem_wait_ld();
        if constexpr (C::SEP_P) {   // S_i may be overwritten by S_i(j+1) from here on
          tc_fence_before();
          mbar_arrive(&s_free[i]);
        }
        if (!tile_unmasked<BN>(p, skv, r0, j)) {
          const int c_lo = key_lo - j * BN, c_hi = key_hi - j * BN;
#pragma unroll
          for (int c = 0; c < BN; ++c) s[c] = (c >= c_lo && c <= c_hi) ? s[c] : -INFINITY;
        }
        // row maximum: four independent chains of three-input max
        // (columns 0-7 start the chains, then 8 columns per step: exactly s[0, BN))
        float mc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) mc[q] = fmaxf(s[2 * q], s[2 * q + 1]);
#pragma unroll
        for (int c = 8; c < BN; c += 8)
#pragma unroll
          for (int q = 0; q < 4; ++q) mc[q] = fmax3(mc[q], s[c + 2 * q], s[c + 2 * q + 1]);
        const float mx = fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]);
        const float m_tile = mx * p.scale_log2;
        float alpha = 1.f;
        if (m_tile > m_ref + kTau) {
          alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_tile);
          l *= alpha;
          m_ref = m_tile;
        }
        if constexpr (!C::SEP_P) rescale_o(j > my_lo, alpha);   // O_i is current: S_i(j) covers P_i V(j-1)
        const float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t nm2 = f2_pack(-mb, -mb);
        uint32_t pk[BN / 2];
        uint64_t sum2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) sum2[q] = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const uint64_t x2 = f2_fma(f2_pack(s[c], s[c + 1]), c2, nm2);
          float x0, x1;
          f2_unpack(x2, x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          sum2[(c / 2) % 4] = f2_add(sum2[(c / 2) % 4], f2_pack(p0, p1));
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        float s0, s1, s2, s3;
        f2_unpack(f2_add(sum2[0], sum2[1]), s0, s1);
        f2_unpack(f2_add(sum2[2], sum2[3]), s2, s3);
        l += (s0 + s1) + (s2 + s3);
        // The exponentials above need nothing from tensor memory; only now must
        // P_i(j-1) V be complete: before O_i is rescaled and (separate P) before
        // P_i is rewritten.  Waiting here hides that product behind them.
        if constexpr (C::SEP_P) {
          if (j > my_lo) {
            ok = mbar_wait(&o_done[i], pv & 1, abort_flag, p.err);
            ++pv;
            if (!__all_sync(0xffffffffu, ok)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
        }
        if constexpr (C::SEP_P) rescale_o(j > my_lo, alpha);
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tmem_st32(p_tmem + 32 * c, pk + 32 * c);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_ready[i]);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 (tcgen05.ld is warp-collective: every lane loads)
      if constexpr (C::SEP_P) {
        ok = mbar_wait(&o_done[i], pv & 1, abort_flag, p.err);
        ++pv;
      } else {
        ok = mbar_wait(&o_done[i], oc & 1, abort_flag, p.err);
        ++oc;
      }
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // a row with no visible key is 0 (and its lse -inf)
      const bool has_keys = key_hi >= max(key_lo, 0);
      const float inv = (has_keys && l > 0.f) ? 1.f / l : 0.f;
      if (p.lse != nullptr && store)   // log(sum_j exp(s_ij * scale)) = (m + log2 l) * ln 2
        p.lse[static_cast<size_t>(it.bh) * p.Sq + r] =
            (has_keys && l > 0.f) ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(o_tmem + 32 * c, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      tc_fence_before();   // this group's O reads precede the next item's first P_i V product
    }
    // if a wait gave up, the remaining rows stay unwritten and the error word records it
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

namespace {
EncodeTiledFn g_encoder = nullptr;

void look_up_encoder() {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encoder = reinterpret_cast<EncodeTiledFn>(ptr);
}

EncodeTiledFn tensor_map_encoder() {
  static pthread_once_t once = PTHREAD_ONCE_INIT;
  pthread_once(&once, look_up_encoder);
  return g_encoder;
}
}  // namespace

bool make_tensor_map_3d(CUtensorMap* m, const void* base, int elem_bytes, int inner, int rows, int planes,
                        int box_inner, int box_rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr || (elem_bytes != 1 && elem_bytes != 2)) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * elem_bytes,
                                 static_cast<cuuint64_t>(rows) * inner * elem_bytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// [planes][rows][D] bf16 tensor, boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int D, int rows, int planes, int box_rows = 128) {
  return make_tensor_map_3d(m, base, 2, D, rows, planes, 64, box_rows);
}

}  // namespace

int sm_count() {
  constexpr int kMaxDevices = 64;
  static int cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {

// One-time set-up of a kernel on the current device: its shared-memory limit,
// and the check that setmaxnreg.inc can be honoured (it waits until the
// block's own registers cover the request, so a build whose launch
// allocation could not is refused).  Done once per device; later calls skip
// the runtime queries, which cost more host time than the launch itself.
template <int D, bool PAGED>
cudaError_t prepare_kernel() {
  using C = Cfg<D>;
  constexpr int kMaxDevices = 64;
  static int ready[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (__atomic_load_n(&ready[dev], __ATOMIC_ACQUIRE) == 1) return cudaSuccess;
  auto kern = prefill_tc_kernel<D, PAGED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa{};
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * C::THREADS < 128 * (2 * C::SOFTMAX_REGS + C::PRODUCER_REGS))
    return cudaErrorInvalidConfiguration;
  __atomic_store_n(&ready[dev], 1, __ATOMIC_RELEASE);
  return cudaSuccess;
}

template <int D, bool PAGED>
cudaError_t launch_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p,
                     cudaStream_t stream) {
  using C = Cfg<D>;
  auto kern = prefill_tc_kernel<D, PAGED>;
  const size_t smem = C::SMEM;
  cudaError_t e = prepare_kernel<D, PAGED>();
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(min(p.n_items, sms));
  return launch_dependent(kern, dim3(grid), dim3(C::THREADS), smem, stream, mq, mk, mv, p);
}

}  // namespace

cudaError_t launch_prefill_tc(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq,
                              int Hkv, int Sq, int Skv, int D, float scale, int causal, int window, unsigned int* err,
                              cudaStream_t stream) {
  const int bn = (D == 64) ? Cfg<64>::BN : Cfg<128>::BN;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, Sq, B * Hq) || !make_map(&mk, k, D, Skv, B * Hkv, bn) ||
      !make_map(&mv, v, D, Skv, B * Hkv, bn))
    return cudaErrorInvalidValue;
  Params p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.causal = causal;
  p.window = window;
  p.n_qblocks = (Sq + NQ * BM - 1) / (NQ * BM);
  const long long items = static_cast<long long>(p.n_qblocks) * B * Hq;
  if (items > (1LL << 30)) return cudaErrorInvalidValue;
  p.n_items = static_cast<int>(items);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.err = err;
  return D == 64 ? launch_d<64, false>(mq, mk, mv, p, stream) : launch_d<128, false>(mq, mk, mv, p, stream);
}

cudaError_t launch_prefill_tc_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* page_table,
                                    const int32_t* seq_lens, int page_size, int B, int Hq, int Hkv, int Sq, int D,
                                    int num_pages, int max_pages, int max_seq_len, float scale, int causal,
                                    int window, void* out, float* lse, unsigned int* err, cudaStream_t stream) {
  const int bn = (D == 64) ? Cfg<64>::BN : Cfg<128>::BN;
  const int box_rows = page_size < bn ? page_size : bn;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, Sq, B * Hq) || !make_map(&mk, k_pool, D, page_size, num_pages * Hkv, box_rows) ||
      !make_map(&mv, v_pool, D, page_size, num_pages * Hkv, box_rows))
    return cudaErrorInvalidValue;
  Params p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Skv = max_seq_len;
  p.causal = causal;
  p.window = window;
  p.n_qblocks = (Sq + NQ * BM - 1) / (NQ * BM);
  const long long items = static_cast<long long>(p.n_qblocks) * B * Hq;
  if (items > (1LL << 30)) return cudaErrorInvalidValue;
  p.n_items = static_cast<int>(items);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.err = err;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.page_size = page_size;
  p.box_rows = box_rows;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  return D == 64 ? launch_d<64, true>(mq, mk, mv, p, stream) : launch_d<128, true>(mq, mk, mv, p, stream);
}

}  // namespace attn
