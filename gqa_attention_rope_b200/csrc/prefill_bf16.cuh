// prefill_bf16.cuh -- grouped-query causal attention with RoPE and the
// cross-document mask on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA computes a 128-row query tile for NH (1 or 2) query heads of the same
// KV group, so every K/V tile brought in by TMA serves both heads (GQA reuse).
//
//   warp 0      TMA producer: Q tiles once per item, then K tiles through a
//               2-stage K ring and V tiles through a 1-stage V ring, issued in
//               the order K0, K1, V0, K2, V1, ..., so each K tile is loaded
//               one tile ahead of its S MMAs and each V tile while the softmax
//               of its tile runs. It also claims the items and publishes each
//               one's fields in a shared-memory ring.
//   warp 1      TMEM owner; one thread issues S_h = Q_h K_j^T (M=128, N=128,
//               K=128; fp32 accumulators in TMEM)
//   warp 2      one thread issues O_h += P_h V_j (P from shared memory, V MN-major).
//               Two issuing threads: a tcgen05.mma issue blocks at the tensor
//               rate and every barrier wait (~250+ cycles even when the phase
//               has completed) would otherwise leave the tensor pipe idle; with
//               S and PV issued from different threads one thread's waits
//               overlap the other's MMAs.
//   warp 3      one thread stores each finished output tile with TMA.
//   warps 4-7   softmax for head slot 0, warps 8-11 for slot 1: thread = query
//               row = TMEM lane. Rotates its Q row in shared memory (RoPE at the
//               row's document position), then per KV tile: S from TMEM ->
//               registers, mask, row max, P = 2^(S*log2e/sqrt(D) - m) in bf16 to
//               shared memory, running sum; O in TMEM is rescaled only when the
//               running max grows by more than 2^8 (exact: the final 1/l uses the
//               same reference max); epilogue O/l -> bf16 -> TMA store.
//   Registers: the four role warps (one warpgroup) hold 64 each and give the
//   rest to the eight softmax warps, which hold 216 each (setmaxnreg).
//
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
// Shared memory (1024-aligned): Q_0, Q_1 (32 KB each), K ring 2 x 32 KB, V ring
// 32 KB, P_0, P_1 (32 KB each), barriers and the item ring. Every 32 KB tile is
// two 64-column halves of 128 rows x 128 B in the 128B-swizzled layout TMA
// writes.
//
// Items run heaviest first (the last query tiles first); when the keys and
// values are far larger than L2 they run KV group by KV group instead, heaviest
// first inside each group (see item_of).
//
// KV tiles run from the tile holding the document start of the first query
// row to the diagonal tile; tiles entirely before that start are never loaded
// or multiplied. Only tiles on the diagonal or before the last row's document
// start apply the element mask.
//
// Keys arrive already rotated (a separate streaming pass writes RoPE(K) once
// per key, which is cheaper than re-rotating every K tile for every query tile
// that reads it).
#pragma once

#include "ptx.cuh"
#include "rope.cuh"

namespace la {
namespace pfx {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NSTAGE = 3;  // 32 KB ring stages, K and V rings together
constexpr uint32_t TILE = 32768;
constexpr uint32_t HALF = 16384;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_KV = OFF_Q + 2 * TILE;
constexpr uint32_t OFF_P = OFF_KV + NSTAGE * TILE;
constexpr uint32_t OFF_BAR = OFF_P + 2 * TILE;
constexpr uint32_t SMEM_USED = OFF_BAR + 1024;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;
constexpr int NTHREADS = 384;
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleLog2 = 8.0f;

// K tiles go through a ring of NK stages and V tiles through a ring of NV
// stages (in that order in the ring area); each stage has a full barrier (the
// TMA load's bytes landed) and an empty barrier (the MMAs that read it
// completed). The S issuer waits only on the K ring's full barriers and the PV
// issuer only on the V ring's, each in consecutive phases (tile count /
// stages), so a wait can neither alias nor pass early whatever order separate
// TMA loads land in. Of the splits of the three 32 KB stages, two K stages and
// one V stage measured best: a V tile is needed a whole softmax after its K.
constexpr int NK = 2, NV = 1;
enum : int {
  B_K_FULL = 0,
  B_K_EMPTY = B_K_FULL + NK,
  B_V_FULL = B_K_EMPTY + NK,
  B_V_EMPTY = B_V_FULL + NV,
  B_Q_FULL = B_V_EMPTY + NV,
  B_Q_READY,
  B_S_READY = B_Q_READY + 2,
  B_S_FREE = B_S_READY + 2,
  B_P_READY = B_S_FREE + 2,
  B_PV_DONE = B_P_READY + 2,
  B_O_STAGED = B_PV_DONE + 2,
  B_O_READ = B_O_STAGED + 2,
  B_Q_FREE = B_O_READ + 2,
  B_DRAIN,
  B_DRAIN_PV,
  N_BARS
};
constexpr int kItemRing = 8;
static_assert(N_BARS * 8 + 8 + 8 * kItemRing <= 512, "barrier area, TMEM address and item ring");
// Each ring slot also holds its item's fields, computed once by the producer.
struct ItemSlot {
  int b, h0, g, q0, ds_last, kv_t0, n_kv, pad;
};
constexpr uint32_t OFF_SLOTS = 512;  // from OFF_BAR
static_assert(OFF_SLOTS + sizeof(ItemSlot) * kItemRing <= 1024, "item slots");

struct Params {
  int B, S, Hq, Hkv, G, NH, n_qt, n_hp;
  // Key/value rows per batch row (S unless the queries are chunks of a longer
  // sequence) and RoPE table rows (max(S, Skv)).
  int Skv, n_pos;
  // Global position of local query row 0 and of local row q_split (a multiple
  // of 128; S when all rows form one chunk). Both 0 for a plain prefill.
  int q_split, q_pos_a, q_pos_b;
  int q_rotated;             // 1: q arrives already rotated (no in-kernel rotation, no table)
  int kv_major;              // 1: items run KV group by KV group (keys and values far larger than L2)
  const int32_t* doc_start;  // [B*S] row-local document start, or null (one document per row)
  const float4* rope_tab;    // (cos, sin) pairs, 64 per position, as float4 = 2 pairs
  int* sched;                // work-item counter, zero at launch
  float* lse;                // optional [B*S, Hq] log-sum-exp of each row's visible scaled scores
  float scale_log2;          // log2(e) / sqrt(D)
  unsigned int epoch;        // launch id for bounded-wait abort propagation
};

__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return umma_desc_sw128(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t vdesc(uint32_t saddr) { return umma_desc_sw128(saddr, HALF, 1024); }

// One work item: a 128-row query tile of batch row b for query heads
// h0 .. h0 + NH - 1 (all of KV group g). item_of numbers them heaviest first
// (highest query tile first), over all groups or inside each KV group in turn;
// the producer computes each item's fields once and publishes them.
struct Item {
  int b, h0, g, q0, ds_last, kv_t0, n_kv;
  int64_t rowbase;
};

// Global position of local query row q0 (a multiple of 128).
__device__ __forceinline__ int q_global(int q0, const Params& p) {
  return (q0 < p.q_split) ? p.q_pos_a + q0 : p.q_pos_b + (q0 - p.q_split);
}

__device__ __forceinline__ Item item_of(int item, const Params& p) {
  Item it;
  int qt;
  if (p.kv_major) {
    // By (batch row, KV group) block, inside a block from the last (heaviest)
    // query tile down, head pair by head pair: the CTAs at work at any time
    // read one KV group's keys and values, which then stay in L2.
    const int pg = p.G / p.NH;  // head pairs (or single heads) per KV group
    const int per_blk = p.n_qt * pg;
    const int blk = item / per_blk, rem = item % per_blk;
    it.b = blk / p.Hkv;
    it.g = blk % p.Hkv;
    qt = p.n_qt - 1 - rem / pg;
    it.h0 = (it.g * pg + rem % pg) * p.NH;
  } else {
    // Heaviest first: the last query tile of every batch row and head pair,
    // then the one before, ... (longest-processing-time-first)
    const int per_rank = p.B * p.n_hp;
    qt = p.n_qt - 1 - item / per_rank;
    const int rem = item % per_rank;
    it.b = rem / p.n_hp;
    it.h0 = (rem % p.n_hp) * p.NH;
    it.g = it.h0 / p.G;
  }
  it.q0 = qt * BM;
  const int q_last = min(it.q0 + BM - 1, p.S - 1);
  it.rowbase = static_cast<int64_t>(it.b) * p.S;
  const int ds_first = p.doc_start ? p.doc_start[it.rowbase + it.q0] : 0;
  it.ds_last = p.doc_start ? p.doc_start[it.rowbase + q_last] : 0;
  it.kv_t0 = ds_first / BN;
  it.n_kv = q_global(it.q0, p) / BN - it.kv_t0 + 1;  // the last tile holds the diagonal
  return it;
}

// Persistent: one CTA per SM. Its first item is blockIdx.x; later ones are
// claimed with an atomic counter (gridDim.x + counter), so items are handed
// out first-come in item_of's order (longest-processing-time-first, inside each
// KV group when the items run group by group).
// The producer publishes each claimed item id in an 8-entry shared-memory ring
// as soon as it is claimed (well before its Q tiles are loaded); -1 ends every
// role's loop.
// The ring counters and the per-tile barrier phases run on across items; the
// next item's Q tiles are loaded as soon as the S MMAs of the current item have
// finished reading Q, and the output tile is staged in the P buffer and stored
// by warp 3, so one item's tail overlaps the next item's start.
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * N_BARS);
  // item ring: slot k holds (item id, sequence number); the producer writes the
  // item, then the sequence number; readers poll the sequence number.
  volatile int* ring_item = reinterpret_cast<volatile int*>(smem + OFF_BAR + 8 * N_BARS + 8);
  volatile int* ring_seq = ring_item + kItemRing;
  volatile ItemSlot* slots = reinterpret_cast<volatile ItemSlot*>(smem + OFF_BAR + OFF_SLOTS);
  // The item published in ring slot k (read once its sequence number, or a
  // barrier phase that follows the publication, has been seen).
  auto slot_item = [&](int k) -> Item {
    const volatile ItemSlot& q = slots[k % kItemRing];
    Item it;
    it.b = q.b;
    it.h0 = q.h0;
    it.g = q.g;
    it.q0 = q.q0;
    it.ds_last = q.ds_last;
    it.kv_t0 = q.kv_t0;
    it.n_kv = q.n_kv;
    it.rowbase = static_cast<int64_t>(it.b) * p.S;
    return it;
  };
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{p.epoch};
  const int n_items = p.B * p.n_qt * p.n_hp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(bar(B_K_FULL + s), 1);
      mbar_init(bar(B_K_EMPTY + s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bar(B_V_FULL + s), 1);
      mbar_init(bar(B_V_EMPTY + s), 1);
    }
    mbar_init(bar(B_Q_FULL), 1);
    mbar_init(bar(B_Q_FREE), 2);  // the S issuer's commit and the PV issuer's arrival
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_Q_READY + s), 128);
      mbar_init(bar(B_S_READY + s), 1);
      mbar_init(bar(B_S_FREE + s), 128);
      mbar_init(bar(B_P_READY + s), 128);
      mbar_init(bar(B_PV_DONE + s), 1);
      mbar_init(bar(B_O_STAGED + s), 128);
      mbar_init(bar(B_O_READ + s), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_DRAIN_PV), 1);
    for (int k = 0; k < kItemRing; ++k) {  // no slot may look published before it is
      ring_seq[k] = -1;
      ring_item[k] = -1;
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Registers: the role warpgroup (warps 0-3) gives up registers to the two
  // softmax warpgroups: 64 * 128 + 2 * 216 * 128 = 63,488, within the launch's
  // 384 threads x 168 = 64,512. Each setmaxnreg heads its warpgroup's branch, so the
  // compiler allocates every role's code for the count that warpgroup holds.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        uint32_t kt = 0, vt = 0;  // K and V tiles loaded so far
        bool ok = true;
        // One tile into stage (count % n) of its ring, after the stage's previous
        // tile has been consumed (empty barrier, phase count / n - 1).
        auto load_tile = [&](const CUtensorMap* tm, uint32_t& count, int n, int b_full, int b_empty, uint32_t off,
                             int g, int kv_row, int b) -> bool {
          const uint32_t st = count % n, use = count / n;
          if (use > 0 && !mbar_wait_backoff(bar(b_empty + st), (use - 1) & 1, wc)) return false;
          const uint32_t full = bar(b_full + static_cast<int>(st));
          mbar_arrive_expect_tx(full, TILE);
          tma_load_4d(sbase + off + st * TILE, tm, full, 0, g, kv_row, b);
          tma_load_4d(sbase + off + st * TILE + HALF, tm, full, 64, g, kv_row, b);
          ++count;
          return true;
        };
        auto load_k = [&](int g, int kv_row, int b) {
          return load_tile(&tm_k, kt, NK, B_K_FULL, B_K_EMPTY, OFF_KV, g, kv_row, b);
        };
        auto load_v = [&](int g, int kv_row, int b) {
          return load_tile(&tm_v, vt, NV, B_V_FULL, B_V_EMPTY, OFF_KV + NK * TILE, g, kv_row, b);
        };
        // The RoPE table rows an item's Q rotation will read: positions
        // q0 - ds(q0) .. +127 and, when a document starts inside the tile, 0 .. 127.
        auto prefetch_rows = [&](int v) {
          if (v < 0 || v >= n_items || p.q_rotated) return;
          const Item J = item_of(v, p);
          const int ds0 = p.doc_start ? p.doc_start[J.rowbase + J.q0] : 0;
          const int p0 = q_global(J.q0, p) - ds0;
          const int n0 = min(BM, p.n_pos - p0);
          if (n0 > 0) bulk_prefetch_l2(p.rope_tab + static_cast<int64_t>(p0) * 32, static_cast<uint32_t>(n0) * 512u);
          if (J.ds_last > J.q0) bulk_prefetch_l2(p.rope_tab, static_cast<uint32_t>(min(BM, p.n_pos)) * 512u);
        };
        auto publish = [&](int k, int v) {
          if (v >= 0 && v < n_items) {
            const Item J = item_of(v, p);
            volatile ItemSlot& q = slots[k % kItemRing];
            q.b = J.b;
            q.h0 = J.h0;
            q.g = J.g;
            q.q0 = J.q0;
            q.ds_last = J.ds_last;
            q.kv_t0 = J.kv_t0;
            q.n_kv = J.n_kv;
          }
          ring_item[k % kItemRing] = v;
          __threadfence_block();
          ring_seq[k % kItemRing] = k;
        };
        int it = 0, item = blockIdx.x;
        int next_item = (item < n_items) ? atomicAdd(p.sched, 1) + static_cast<int>(gridDim.x) : n_items;
        bool ended = false;
        publish(0, item < n_items ? item : -1);
        prefetch_rows(item);
        for (;; ++it) {
          if (it > 0 && !mbar_wait_backoff(bar(B_Q_FREE), (it - 1) & 1, wc)) {
            ok = false;
            break;
          }
          if (item >= n_items) {
            mbar_arrive(bar(B_Q_FULL));
            ended = true;
            break;
          }
          const Item I = slot_item(it);
          mbar_arrive_expect_tx(bar(B_Q_FULL), static_cast<uint32_t>(p.NH) * TILE);
          for (int s = 0; s < p.NH; ++s)
            for (int hf = 0; hf < 2; ++hf)
              tma_load_4d(sbase + OFF_Q + s * TILE + hf * HALF, &tm_q, bar(B_Q_FULL), hf * 64, I.h0 + s, I.q0, I.b);
          // The item's first K tiles go out before the next item is claimed and
          // published (an atomic and two document-start reads): the first S
          // MMAs wait for them, the consumers of the next item's fields not yet.
          ok = load_k(I.g, I.kv_t0 * BN, I.b);
          if (ok && I.n_kv > 1) ok = load_k(I.g, (I.kv_t0 + 1) * BN, I.b);
          item = next_item;
          next_item = (item < n_items) ? atomicAdd(p.sched, 1) + static_cast<int>(gridDim.x) : n_items;
          publish(it + 1, item < n_items ? item : -1);
          prefetch_rows(item);
          if (ok && I.n_kv > 1) ok = load_v(I.g, I.kv_t0 * BN, I.b);
          for (int j = 2; ok && j < I.n_kv; ++j)
            ok = load_k(I.g, (I.kv_t0 + j) * BN, I.b) && load_v(I.g, (I.kv_t0 + j - 1) * BN, I.b);
          if (ok) ok = load_v(I.g, (I.kv_t0 + I.n_kv - 1) * BN, I.b);
          if (!ok) {
            ++it;
            break;
          }
        }
        // Every issued load has landed before this CTA may exit (these return at
        // once in the normal flow, where every load was consumed).
        if (!ended && it > 0) mbar_wait(bar(B_Q_FULL), (it - 1) & 1, wc);
        // Only the last tile into a stage can still be in flight (each load
        // waited for the stage to be emptied): wait for the latest phase of each.
        for (uint32_t st = 0; st < NK; ++st)
          if (kt > st) mbar_wait(bar(B_K_FULL + static_cast<int>(st)), ((kt - 1 - st) / NK) & 1, wc);
        for (uint32_t st = 0; st < NV; ++st)
          if (vt > st) mbar_wait(bar(B_V_FULL + static_cast<int>(st)), ((vt - 1 - st) / NV) & 1, wc);
      }
    } else if (warp == 1 || warp == 2) {
      // ------------------------------------------------------------ MMA issuers
      // Tile T (counted over all items) sits in K stage T % NK and V stage
      // T % NV, loaded there for the (T / NK)-th and (T / NV)-th time.
      if (lane == 0) {
        constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(128, 128, 0);
        constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(128, 128, 1);
        bool ok = true;
        uint32_t tiles = 0;

        for (int it = 0; ok; ++it) {
          if (!mbar_wait(bar(B_Q_FULL), it & 1, wc)) break;
          // The PV issuer waits on Q_FULL only to learn the item id; its arrival
          // on Q_FREE keeps the next Q load behind this wait, so its parity wait
          // can never fall two phases behind.
          if (warp == 2) mbar_arrive(bar(B_Q_FREE));
          const int item = ring_item[it % kItemRing];
          if (item < 0 || item >= n_items) break;
          const Item I = slot_item(it);
          if (warp == 1) {
            for (int s = 0; s < p.NH; ++s) ok = ok && mbar_wait(bar(B_Q_READY + s), it & 1, wc);
            for (int j = 0; ok && j < I.n_kv; ++j) {
              const uint32_t T = tiles + j;  // K tile count = tile count
              const uint32_t st = T % NK;
              if (!mbar_wait(bar(B_K_FULL + static_cast<int>(st)), (T / NK) & 1, wc)) {
                ok = false;
                break;
              }
              const uint64_t db = kdesc(sbase + OFF_KV + st * TILE);
              for (int s = 0; s < p.NH; ++s) {
                if (T > 0 && !mbar_wait(bar(B_S_FREE + s), (T - 1) & 1, wc)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint64_t da = kdesc(sbase + OFF_Q + s * TILE);
  #pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint64_t off = ((kk >> 2) * HALF + (kk & 3) * 32) >> 4;
                  tc_mma_ss(tmem + s * 128, da + off, db + off, idesc_qk, kk > 0);
                }
                tc_commit(bar(B_S_READY + s));
              }
              tc_commit(bar(B_K_EMPTY + static_cast<int>(st)));
            }
            tc_commit(bar(B_Q_FREE));  // the Q tiles are free once these MMAs complete
          } else {
            for (int j = 0; ok && j < I.n_kv; ++j) {
              const uint32_t T = tiles + j;  // V tile count = tile count
              const uint32_t st = T % NV;
              if (!mbar_wait(bar(B_V_FULL + static_cast<int>(st)), (T / NV) & 1, wc)) {
                ok = false;
                break;
              }
              const uint64_t db = vdesc(sbase + OFF_KV + (NK + st) * TILE);
              for (int s = 0; s < p.NH; ++s) {
                if (!mbar_wait(bar(B_P_READY + s), T & 1, wc)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint64_t da = kdesc(sbase + OFF_P + s * TILE);
  #pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint64_t aoff = ((kk >> 2) * HALF + (kk & 3) * 32) >> 4;
                  tc_mma_ss(tmem + 256 + s * 128, da + aoff, db + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                            (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar(B_PV_DONE + s));
              }
              tc_commit(bar(B_V_EMPTY + static_cast<int>(st)));
            }
          }
          tiles += static_cast<uint32_t>(I.n_kv);
        }
        // all issued MMAs complete before TMEM may be freed
        const int drain = (warp == 1) ? B_DRAIN : B_DRAIN_PV;
        tc_commit(bar(drain));
        mbar_wait(bar(drain), 0, wc);
      }
    } else if (warp == 3) {
      // ------------------------------------------------------------ output stores
      if (lane == 0) {
        bool ok = true;
        for (int it = 0; ok; ++it) {
          if (!mbar_wait_backoff(bar(B_O_STAGED + 0), it & 1, wc)) break;
          const int item = ring_item[it % kItemRing];
          if (item < 0 || item >= n_items) break;
          const Item I = slot_item(it);
          for (int s = 0; ok && s < p.NH; ++s) {
            if (s > 0 && !mbar_wait_backoff(bar(B_O_STAGED + s), it & 1, wc)) {
              ok = false;
              break;
            }
            tma_store_4d(&tm_o, sbase + OFF_P + s * TILE, 0, I.h0 + s, I.q0, I.b);
            tma_store_4d(&tm_o, sbase + OFF_P + s * TILE + HALF, 64, I.h0 + s, I.q0, I.b);
            tma_store_commit();
            tma_store_wait_read0();  // the P buffer may be rewritten from here on
            mbar_arrive(bar(B_O_READ + s));
          }
        }
        tma_store_wait0();
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;");
    if ((warp - 4) / 4 < p.NH) {
      // ------------------------------------------------------------ softmax
      const int s = (warp - 4) >> 2;
      const int wq = warp & 3;
      const int r = wq * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
      const uint32_t tS = tmem + lane_off + s * 128;
      const uint32_t tO = tmem + lane_off + 256 + s * 128;
      uint8_t* qtile = smem + OFF_Q + s * TILE;
      uint8_t* ptile = smem + OFF_P + s * TILE;
      const float sl2 = p.scale_log2;
      bool ok = true;
      uint32_t tiles = 0;
      Item I;
      int qi_c = 0, ds_i = 0;  // global position of this thread's (clamped) row; its document start
      // Starts item `it`: reads its id from the ring, loads its row data, waits for
      // its Q tile and rotates this thread's row in place. False at the end of the
      // items (or on a timeout, which also clears ok).
      auto begin_item = [&](int it) -> bool {
        int item = -1;
        {
          const unsigned long long t0 = global_ns();
          for (uint32_t k = 0;; ++k) {
            if (ring_seq[it % kItemRing] == it) {
              __threadfence_block();  // the item id was written before its sequence number
              item = ring_item[it % kItemRing];
              break;
            }
            if ((k & 63u) == 63u && (wc.aborted() || global_ns() - t0 > kWaitTimeoutNs)) {
              if (!wc.aborted()) {
                raise_error(LLAMA_ATTN_DEVERR_TIMEOUT);
                atomicExch(&g_abort_epoch, wc.epoch);
              }
              ok = false;
              return false;
            }
          }
        }
        if (item < 0) return false;
        if (item >= n_items) {  // cannot happen unless the ring protocol is broken
          raise_error(LLAMA_ATTN_DEVERR_TIMEOUT);
          atomicExch(&g_abort_epoch, wc.epoch);
          ok = false;
          return false;
        }
        I = slot_item(it);
        const int qi = I.q0 + r;
        qi_c = min(qi, p.S - 1);
        ds_i = p.doc_start ? p.doc_start[I.rowbase + qi_c] : 0;
        qi_c += q_global(I.q0, p) - I.q0;  // from here on the row's global position
        if (!mbar_wait(bar(B_Q_FULL), it & 1, wc)) {
          ok = false;
          return false;
        }
        // Rotate the warp's 32 Q rows two at a time: 16 lanes per row, 4 pairs
        // per lane. A half-warp walks rows 2 apart; inside a document their
        // positions are 2 apart too, so the (cos, sin) of the next row follow
        // from the current ones by one rotation by 2*theta_k (angle addition,
        // the table's row for position 2). The table is read only for the first
        // row and where positions restart at a document start.
        if (!p.q_rotated) {
          const int ch = lane & 15;
          const float4* step = p.rope_tab + 2 * 32 + 2 * ch;
          const float4 st0 = __ldg(step), st1 = __ldg(step + 1);
          float4 c0 = make_float4(1.f, 0.f, 1.f, 0.f), c1 = c0;
          int pos_prev = -4;
          const int pos_own = qi_c - ds_i;
          const uint32_t hoff = (ch >> 3) * HALF;
          // Four of the half-warp's rows at a time: their chunks are all read
          // before any is written back, so one shared-memory round trip (slow
          // here: the last PV MMAs and the next item's TMA loads share the
          // bandwidth) serves four rows.
  #pragma unroll 1
          for (int i0 = 0; i0 < 16; i0 += 4) {
            uint4 x[4];
  #pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int rr = wq * 32 + 2 * (i0 + u) + (lane >> 4);
              x[u] = *reinterpret_cast<const uint4*>(qtile + hoff + sw128_off(rr, ch & 7));
            }
  #pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int src = 2 * (i0 + u) + (lane >> 4);  // lane of the warp that owns the row
              const int pos = __shfl_sync(0xffffffffu, pos_own, src);
              if (pos == pos_prev + 2) {
                c0 = make_float4(c0.x * st0.x - c0.y * st0.y, c0.y * st0.x + c0.x * st0.y,
                                 c0.z * st0.z - c0.w * st0.w, c0.w * st0.z + c0.z * st0.w);
                c1 = make_float4(c1.x * st1.x - c1.y * st1.y, c1.y * st1.x + c1.x * st1.y,
                                 c1.z * st1.z - c1.w * st1.w, c1.w * st1.z + c1.z * st1.w);
              } else {
                const float4* tab = p.rope_tab + static_cast<int64_t>(pos) * 32 + 2 * ch;
                c0 = __ldg(tab);
                c1 = __ldg(tab + 1);
              }
              pos_prev = pos;
              x[u].x = rope_rotate_pair(x[u].x, c0.x, c0.y);
              x[u].y = rope_rotate_pair(x[u].y, c0.z, c0.w);
              x[u].z = rope_rotate_pair(x[u].z, c1.x, c1.y);
              x[u].w = rope_rotate_pair(x[u].w, c1.z, c1.w);
            }
  #pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int rr = wq * 32 + 2 * (i0 + u) + (lane >> 4);
              if (I.q0 + rr < p.S) *reinterpret_cast<uint4*>(qtile + hoff + sw128_off(rr, ch & 7)) = x[u];
            }
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_Q_READY + s));
        return true;
      };

      bool more = begin_item(0);
      const bool begin_ok_first = more;
      for (int it = 0; ok && more; ++it) {
        float m = -INFINITY;  // reference max, in log2 units of the scaled score
        float l = 0.f;
        for (int j = 0; j < I.n_kv; ++j) {
          const int kb = (I.kv_t0 + j) * BN;
          const uint32_t T = tiles + j;
          if (!mbar_wait(bar(B_S_READY + s), T & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t sr[128];
          tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
          tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
          tc_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(B_S_FREE + s));

          float sv[128];
  #pragma unroll
          for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(sr[c]);
          if (j == I.n_kv - 1 || kb < I.ds_last) {  // the diagonal tile, or a document starts in it
            const int lo = ds_i - kb, hi = qi_c - kb;
  #pragma unroll
            for (int c = 0; c < 128; ++c) sv[c] = (c < lo || c > hi) ? -INFINITY : sv[c];
          }
          // four running maxima over columns a, a+4, ..., a+124 (a = 0..3)
          float mx0 = sv[0], mx1 = sv[1], mx2 = sv[2], mx3 = sv[3];
  #pragma unroll
          for (int c = 4; c <= 116; c += 8) {
            mx0 = max3(mx0, sv[c], sv[c + 4]);
            mx1 = max3(mx1, sv[c + 1], sv[c + 5]);
            mx2 = max3(mx2, sv[c + 2], sv[c + 6]);
            mx3 = max3(mx3, sv[c + 3], sv[c + 7]);
          }
          mx0 = fmaxf(mx0, sv[124]);
          mx1 = fmaxf(mx1, sv[125]);
          mx2 = fmaxf(mx2, sv[126]);
          mx3 = fmaxf(mx3, sv[127]);
          const float mt = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
          const float m_new = fmaxf(m, mt);
          const bool resc = m_new > m + kRescaleLog2;
          float alpha = 1.f;
          if (resc) {
            alpha = ex2_approx(m - m_new);
            m = m_new;
          }
          const float neg_m = (m == -INFINITY) ? 0.f : -m;
          uint32_t pk[64];
          // x = s * log2(e)/sqrt(D) - m and the running row sum in packed fp32 pairs
          const uint64_t sl2x2 = f2_pack(sl2, sl2), negmx2 = f2_pack(neg_m, neg_m);
          uint64_t rsa = f2_pack(0.f, 0.f), rsb = rsa;
  #pragma unroll
          for (int c = 0; c < 128; c += 2) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(sv[c], sv[c + 1]), sl2x2, negmx2), x0, x1);
            // one pair in sixteen goes through the FMA-pipe polynomial, the rest
            // through MUFU (1/16 measured best on all three prefill workloads,
            // 1/8 within 1.5%; 1/4 and larger shares cost more FMA and ALU
            // issue than the MUFU time saved)
            const bool poly = (c & 30) == 30;
            const float p0 = poly ? ex2_poly(x0) : ex2_approx(x0);
            const float p1 = poly ? ex2_poly(x1) : ex2_approx(x1);
            if (c & 2) rsb = f2_add(rsb, f2_pack(p0, p1));
            else rsa = f2_add(rsa, f2_pack(p0, p1));
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
          float rs0, rs1, rs2, rs3;
          f2_unpack(rsa, rs0, rs1);
          f2_unpack(rsb, rs2, rs3);
          l = l * alpha + ((rs0 + rs2) + (rs1 + rs3));

          if (j > 0) {
            if (!mbar_wait(bar(B_PV_DONE + s), (T - 1) & 1, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, resc)) {
  #pragma unroll
              for (int ch = 0; ch < 4; ++ch) {
                uint32_t o[32];
                tmem_ld32(tO + ch * 32, o);
                tc_wait_ld();
  #pragma unroll
                for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                tmem_st32(tO + ch * 32, o);
              }
              tc_wait_st();
            }
          } else if (it > 0 && !mbar_wait(bar(B_O_READ + s), (it - 1) & 1, wc)) {
            // the previous item's output left the P buffer
            ok = false;
            break;
          }
  #pragma unroll
          for (int c = 0; c < 16; ++c) {
            uint4 w;
            w.x = pk[4 * c];
            w.y = pk[4 * c + 1];
            w.z = pk[4 * c + 2];
            w.w = pk[4 * c + 3];
            *reinterpret_cast<uint4*>(ptile + (c >> 3) * HALF + sw128_off(r, c & 7)) = w;
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(bar(B_P_READY + s));
        }
        if (!ok) break;

        // The next item's Q rotation overlaps the last PV of this one.
        const Item cur = I;
        const float l_cur = l;
        more = begin_item(it + 1);
        if (!ok) break;

        // ---- epilogue: O / l -> bf16 -> P buffer; warp 3 stores it with TMA
        const uint32_t T_last = tiles + cur.n_kv - 1;
        if (!mbar_wait(bar(B_PV_DONE + s), T_last & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float inv_l = 1.f / l_cur;
  #pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o[32];
          tmem_ld32(tO + ch * 32, o);
          tc_wait_ld();
  #pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * c4 + 0]) * inv_l, __uint_as_float(o[8 * c4 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[8 * c4 + 2]) * inv_l, __uint_as_float(o[8 * c4 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[8 * c4 + 4]) * inv_l, __uint_as_float(o[8 * c4 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[8 * c4 + 6]) * inv_l, __uint_as_float(o[8 * c4 + 7]) * inv_l);
            const int d = ch * 32 + c4 * 8;
            *reinterpret_cast<uint4*>(ptile + (d >> 6) * HALF + sw128_off(r, (d & 63) >> 3)) = w;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_O_STAGED + s));
        if (p.lse != nullptr && cur.q0 + r < p.S)  // natural log: ln 2 * (m + log2 l)
          p.lse[(cur.rowbase + cur.q0 + r) * p.Hq + cur.h0 + s] = 0.69314718055994531f * (m + log2f(l_cur));
        tiles += static_cast<uint32_t>(cur.n_kv);
        if (!more && ok && s == 0) {
          // tell the store warp the items are done, once it has read the last output
          mbar_wait(bar(B_O_READ + 0), it & 1, wc);
          mbar_arrive(bar(B_O_STAGED + 0));
        }
      }
      if (ok && s == 0 && !begin_ok_first) mbar_arrive(bar(B_O_STAGED + 0));  // no items at all
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace pfx
}  // namespace la
