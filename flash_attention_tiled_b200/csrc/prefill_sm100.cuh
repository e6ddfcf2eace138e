// prefill_sm100.cuh -- tiled causal/non-causal attention forward on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes is the FlashAttention-style forward of the "Real-time
// inference optimisation" page (llmapi-app.pages.dev), section "Flash
// Attention optimisation": for each query tile, loop over 128-key tiles,
// S = Q.K^T, online softmax (running max and sum, accumulator rescaled when
// the max moves), O += P.V, finally O / l; plus causal masking and MQA/GQA
// from the "FlashRT-HF-kernels" page (zingnex.cn), section "Attention
// optimisation".  Key tiles that the causal mask hides completely are never
// loaded or multiplied.
//
// A work item is two 128-row query tiles A and B that share every K/V tile.
// When a KV head serves an even number of query heads (GQA with g even, MQA)
// the tiles are the same 128 rows of two query heads of one KV head, so each
// K/V tile staged in shared memory serves two heads of its group (the MQA/GQA
// head sharing of the "FlashRT-HF-kernels" page); otherwise (g odd, e.g. MHA)
// they are rows 0-127 and 128-255 of a 256-row block of one head.  The kernel
// is persistent: one CTA per SM walks its items (see prefill_kernel).
// Tensor memory holds S_A, S_B (128 fp32 columns each) and O_A, O_B (D
// columns each).  P_X is written as bf16 into its own shared-memory tile (the
// A operand of O_X += P_X.V), so S_X is free as soon as the softmax has read
// it: S_X(j+1) is computed while the softmax of tile j is still busy.
// Roles (12 warps):
//   warp 0      TMA producer: per item Q_A and Q_B, then K and V tiles into a
//               ring of shared-memory slots (128-byte swizzled), in the
//               order the MMA warp uses them (K0, K1, V0, K2, V1, ...).
//   warp 1      allocates tensor memory and issues every MMA from one
//               thread: per key tile j, S_A(j+1), S_B(j+1) (as soon as the
//               softmax released S), then PV_A(j), PV_B(j) (as soon as P is
//               written).
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: one query row
//               per thread (= one TMEM lane); exp2 domain (scale*log2(e)
//               folded in); then the epilogue (O / l -> bf16 -> shared memory
//               (P's slot) -> TMA store, and the LSE).
// The producer/MMA warpgroup gives registers to the two softmax warpgroups
// (setmaxnreg): 128 x 88 + 256 x 208 = 384 x 168 registers, the launch's pool.
// Rescaling is lazy: the exponent reference only moves when the row max grows
// by more than 2^8, so O is rarely touched; the result is exact either way
// because numerator and denominator share the reference.
#pragma once

#include "frt_device.cuh"

namespace frt {

constexpr int kPfBM = 128;             // query rows per tile (TMEM lanes)
constexpr int kPfBN = 128;             // keys per tile
constexpr int kPfTiles = 2;            // query tiles per CTA
constexpr int kPfRows = kPfBM * kPfTiles;
constexpr int kPfThreads = 384;
constexpr int kPfRegsLaunch = 168;     // 65536 / 384, rounded down to a multiple of 8
constexpr int kPfRegsProducer = 88;    // warpgroup 0 after setmaxnreg.dec
constexpr int kPfRegsSoftmax = 208;    // warpgroups 1, 2 after setmaxnreg.inc
static_assert(128 * kPfRegsProducer + 256 * kPfRegsSoftmax <= kPfThreads * kPfRegsLaunch,
              "register split must fit in the launch's register pool");
constexpr float kPfRescaleThreshold = 8.0f;   // log2 units

template <int D>
struct PrefillSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = 128 * 128;              // 128 rows x 64 bf16
  static constexpr int kTileBytes = kHalves * kHalfBytes;   // a Q, K or V tile
  static constexpr int kPBytes = 128 * kPfBN * 2;          // one P tile (bf16)
  static constexpr int kSlots = (D == 128) ? 3 : 4;         // K/V ring
  static constexpr int kQOff = 0;                           // Q_A, Q_B
  static constexpr int kPOff = kPfTiles * kTileBytes;       // P_A, P_B
  static constexpr int kRingOff = kPOff + kPfTiles * kPBytes;
  static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
  static constexpr int kNumBars = 2 + 2 * kSlots + 4 * kPfTiles + 1 + 1;
  static constexpr int kBytes = 1024 + kBarOff + kNumBars * 8 + 64;
  static_assert(kBytes <= 227 * 1024, "shared memory budget");
  static_assert(kBytes < (1 << 18), "descriptor address field (14 bits of 16-byte units)");
  // TMEM columns: S_A [0,128), S_B [128,256), O_A [256, 256+D), O_B after it
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
  __device__ static constexpr uint32_t col_s(int t) { return t ? kColS1 : kColS0; }
  __device__ static constexpr uint32_t col_o(int t) { return t ? kColO1 : kColO0; }
};

struct PrefillParams {
  float* lse;          // [B, Hq, Sq] or nullptr
  int B, Hq, Hkv, g, Sq, Skv, causal, n_blocks;   // n_blocks = ceil(Sq / block rows)
  int head_pairs;      // 1: the two tiles are two heads (g even), 128-row blocks;
                       // 0: the two tiles are two row halves of one head, 256-row blocks
  int n_items;         // B * (Hq / heads per item) * n_blocks work items
  float scale_log2;
  // paged K/V (chunked prefill): Sq is the padded chunk length max_q, the
  // per-sequence chunk and context lengths are read on the device
  const int32_t* block_table;   // [B, max_pages]
  const int32_t* seq_lens;      // [B] cached tokens, the chunk included
  const int32_t* q_lens;        // [B] chunk lengths (<= Sq)
  int max_pages;
  int num_pages;                // entries outside [0, num_pages) read row bad_row
  int bad_row;                  // rows of the page pool's [rows, D] view (< 2^31): zeros
};

// One work item: two 128-row query tiles of one (sequence, KV head).  Tile t
// covers query head hq0 + t * dh, rows q_blk + t * dr .. + 127.
struct PrefillItem {
  int b, hq0, kvh, q_blk, dh, dr;
  int sq_b, skv_b, off;   // chunk length, context length, bottom-right causal offset
  int n_kv;               // key tiles to visit (0: the item only writes o = 0)
  bool v_tail_fill;       // paged: the last V tile's rows past the sequence end are zeroed
};

// Items are numbered heaviest first (causal: the last query blocks see the
// most keys), the (sequence, head) index running fastest.
template <bool kPaged>
__device__ __forceinline__ PrefillItem prefill_item(const PrefillParams& p, int w) {
  PrefillItem it;
  const int heads_per_item = p.head_pairs ? 2 : 1;
  const int blk_rows = p.head_pairs ? kPfBM : kPfRows;
  const int hgrp = p.Hq / heads_per_item;
  const int x = w % (p.B * hgrp), y = w / (p.B * hgrp);
  const int blk = p.causal ? (p.n_blocks - 1 - y) : y;
  it.b = x / hgrp;
  it.hq0 = (x % hgrp) * heads_per_item;
  it.kvh = it.hq0 / p.g;                // (g even: both heads share it)
  it.dh = p.head_pairs ? 1 : 0;
  it.dr = p.head_pairs ? 0 : kPfBM;
  it.q_blk = blk * blk_rows;
  it.sq_b = p.Sq;
  it.skv_b = p.Skv;
  if (kPaged) {
    it.sq_b = min(max(p.q_lens[it.b], 0), p.Sq);
    it.skv_b = min(max(p.seq_lens[it.b], 0), p.max_pages * 16);
  }
  it.off = it.skv_b - it.sq_b;
  const int q_last = min(it.q_blk + blk_rows - 1, it.sq_b - 1);
  const int n_kv_all = (it.skv_b + kPfBN - 1) / kPfBN;
  it.n_kv = q_last < it.q_blk ? 0 : n_kv_all;   // a block wholly in the padding has no work
  if (p.causal && it.n_kv > 0) {
    const int lim = q_last + it.off;   // largest key any row of the block sees
    it.n_kv = lim < 0 ? 0 : min(n_kv_all, lim / kPfBN + 1);
  }
  it.v_tail_fill = kPaged && it.n_kv > 0 && it.n_kv * kPfBN > it.skv_b;
  return it;
}

// The r-th item of CTA c among G CTAs: rounds of G items, every other round
// dealt in reverse, so the CTAs that took the heaviest items of one round take
// the lightest of the next.  Increasing in r for a fixed c.
__device__ __forceinline__ int prefill_item_index(int r, int c, int G) {
  return r * G + ((r & 1) ? (G - 1 - c) : c);
}

// kPaged: K and V come from a paged cache ([pages, Hkv, 16, D], 2D tensor
// maps over its rows) through the block table, and each sequence has its own
// chunk length q_lens[b] and context length seq_lens[b] (bottom-right causal).
//
// Persistent: one CTA per SM walks its items.  Barrier phases, the K/V ring
// and tensor memory carry over from item to item, so the next item's Q load
// and its first Q.K^T run while the softmax warps finish the current one (its
// last step and its epilogue).  The epilogue stages O in P's shared-memory
// slot, which is free once the last P.V has completed, so Q's slot can take
// the next item's Q as soon as the last Q.K^T has completed.
template <int D, bool kPaged>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const PrefillParams p) {
  using L = PrefillSmem<D>;
  constexpr int kHalves = L::kHalves;
  constexpr int kSlots = L::kSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem + L::kQOff;
  uint8_t* sp = smem + L::kPOff;
  uint8_t* ring = smem + L::kRingOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;                    // Q_A, Q_B of an item landed
  uint64_t* q_empty = q_full + 1;             // every Q.K^T of an item completed
  uint64_t* ring_full = q_empty + 1;
  uint64_t* ring_empty = ring_full + kSlots;
  uint64_t* s_full = ring_empty + kSlots;     // [tile]: QK_X completed
  uint64_t* s_free = s_full + kPfTiles;       // [tile]: S_X read (128 arrivals)
  uint64_t* p_full = s_free + kPfTiles;       // [tile]: P_X written (128 arrivals)
  uint64_t* pv_done = p_full + kPfTiles;      // [tile]: PV_X completed
  uint64_t* mma_drain = pv_done + kPfTiles;
  uint64_t* v_tail = mma_drain + 1;           // paged: last V tile's tail rows zeroed
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int G = (int)gridDim.x, cta = (int)blockIdx.x;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    for (int t = 0; t < kPfTiles; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 128);
      mbar_init(&p_full[t], 128);
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(mma_drain, 1);
    mbar_init(v_tail, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // The set-up above touches no global memory, so it may overlap the kernel
  // before this one in the stream.  Inputs may come from that kernel: wait for
  // it (a no-op unless launched as a programmatic dependent), then let the
  // next kernel get scheduled as this grid's CTAs finish.
  griddep_wait();
  griddep_launch_dependents();

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfRegsProducer));
    if (warp == 0) {
      // ================================================= TMA producer
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
      }
      int slot = 0;
      uint32_t phase = 0;
      bool ok = true;
      int n_done = 0;   // items with key tiles loaded so far (Q phases)
      for (int r = 0; ok; ++r) {
        const int w = prefill_item_index(r, cta, G);
        if (w >= p.n_items) break;
        const PrefillItem it = prefill_item<kPaged>(p, w);
        if (it.n_kv == 0) continue;
        // Q's slots are free once the previous item's last Q.K^T completed
        if (n_done > 0) ok = mbar_wait_warp(q_empty, (uint32_t)((n_done - 1) & 1), &abort_flag);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full, kPfTiles * L::kTileBytes);
#pragma unroll
          for (int t = 0; t < kPfTiles; ++t)
#pragma unroll
            for (int h = 0; h < kHalves; ++h)
              tma_load_4d(sq + t * L::kTileBytes + h * L::kHalfBytes, &tm_q, q_full, h * 64,
                          it.q_blk + t * it.dr, it.hq0 + t * it.dh, it.b);
        }
        // consumption order of the MMA warp: K0, then per key tile j:
        // K_{j+1} (if any), V_j
        auto load = [&](const CUtensorMap* tm, int j) -> bool {
          if (!mbar_wait_warp(&ring_empty[slot], phase ^ 1u, &abort_flag)) return false;
          uint8_t* dst = ring + slot * L::kTileBytes;
          if (!kPaged) {
            if (lane == 0) {
              mbar_arrive_expect_tx(&ring_full[slot], L::kTileBytes);
#pragma unroll
              for (int h = 0; h < kHalves; ++h)
                tma_load_4d(dst + h * L::kHalfBytes, tm, &ring_full[slot], h * 64, j * kPfBN,
                            it.kvh, it.b);
            }
          } else {
            // eight 16-token pages per key tile, each fetched through the
            // block table into its 16 rows of the tile (both column halves)
            const int npg = min(kPfBN / 16, (it.skv_b + 15) / 16 - j * (kPfBN / 16));
            int row = 0;
            if (lane < npg) {
              // an entry outside [0, num_pages) is never an address: the copy
              // starts past the pool's last row (zeros) and the error word
              // records it; valid rows are below 2^31 (checked by the host)
              const int phys =
                  p.block_table[(size_t)it.b * p.max_pages + j * (kPfBN / 16) + lane];
              if ((unsigned)phys < (unsigned)p.num_pages) {
                row = (int)(((long long)phys * p.Hkv + it.kvh) * 16);
              } else {
                row = p.bad_row;
                raise_error(kErrBadPage);
              }
            }
            if (lane == 0) mbar_arrive_expect_tx(&ring_full[slot], npg * kHalves * 16 * 128);
            __syncwarp();
            if (lane < npg) {
#pragma unroll
              for (int h = 0; h < kHalves; ++h)
                tma_load_2d(dst + h * L::kHalfBytes + lane * 16 * 128, tm, &ring_full[slot],
                            h * 64, row);
            }
            if (tm == &tm_v && j == it.n_kv - 1 && it.v_tail_fill) {
              // rows past the sequence end may hold anything (NaN); P is 0
              // there but 0 * NaN is not, so they are zeroed before P.V
              if (!mbar_wait_warp(&ring_full[slot], phase, &abort_flag)) return false;
              const int valid = it.skv_b - j * kPfBN;
              const int chunks = (kPfBN - valid) * 8 * kHalves;   // 16-byte chunks
              for (int i = lane; i < chunks; i += 32) {
                const int h = i / ((kPfBN - valid) * 8);
                const int rem = i % ((kPfBN - valid) * 8);
                *reinterpret_cast<uint4*>(dst + h * L::kHalfBytes + (valid + rem / 8) * 128 +
                                          (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(v_tail);
            }
          }
          if (++slot == kSlots) { slot = 0; phase ^= 1u; }
          return true;
        };
        ok = load(&tm_k, 0);
        for (int j = 0; j < it.n_kv && ok; ++j) {
          if (j + 1 < it.n_kv) ok = load(&tm_k, j + 1);
          if (ok) ok = load(&tm_v, j);
        }
        ++n_done;
      }
      if (!ok) __nanosleep(100000);
    } else if (warp == 1 && lane == 0) {
      // ===================================================== MMA issuer
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kPfBM, kPfBN, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(kPfBM, D, false, true);
      const uint32_t sq_addr = smem_u32(sq);
      const uint32_t ring_addr = smem_u32(ring);
      int slot = 0;
      uint32_t phase = 0;
      bool ok = true;
      int n_done = 0;   // items with key tiles issued so far (Q phases)
      int n_s = 0;      // S_X computed so far, over all items (s_free phases)
      int n_pv = 0;     // P_X.V issued so far, over all items (p_full phases)
      int n_vt = 0;     // items whose last V tile had its tail zeroed (v_tail phases)

      // This thread sits on the tensor pipe's critical path: the fewer
      // instructions between two MMAs, the less the pipe idles.  So each
      // operand's descriptor is formed once per chain and a K-step's is that
      // base plus the step's offset in 16-byte units (the address field
      // cannot carry: shared-memory addresses are below 2^18).  The bases pass
      // through opaque_int so that they are formed at each chain instead of
      // hoisted out of the loops and held in registers.
      auto issue_qk = [&](int t, uint32_t k_addr) {
        const uint64_t qd = umma_desc_sw128(opaque_int(sq_addr + t * L::kTileBytes), 16, 1024);
        const uint64_t kd = umma_desc_sw128(opaque_int(k_addr), 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = ((ks >> 2) * L::kHalfBytes + (ks & 3) * 32) >> 4;
          tc_mma_ss(tmem + L::col_s(t), qd + koff, kd + koff, idesc_qk, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, uint32_t v_addr, bool accumulate) {
        const uint64_t pd = umma_desc_sw128(opaque_int(smem_u32(sp) + t * L::kPBytes), 16, 1024);
        const uint64_t vd = umma_desc_sw128(opaque_int(v_addr), L::kHalfBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < kPfBN / 16; ++kk) {
          const uint32_t poff = ((kk >> 2) * L::kHalfBytes + (kk & 3) * 32) >> 4;
          tc_mma_ss(tmem + L::col_o(t), pd + poff, vd + kk * (2048 >> 4), idesc_pv,
                    (accumulate || kk > 0) ? 1u : 0u);
        }
        tc_commit(&pv_done[t]);
      };
      auto next_slot = [&]() {
        if (++slot == kSlots) { slot = 0; phase ^= 1u; }
      };
      // S_A, S_B from the K tile in the current slot, each as soon as the
      // softmax has read the previous S of its tile (from this item or the
      // one before); the item's Q slots are released after its last one
      auto issue_s = [&](bool last_of_item) -> bool {
        if (!mbar_wait(&ring_full[slot], phase, &abort_flag)) return false;
        const uint32_t k_addr = ring_addr + slot * L::kTileBytes;
#pragma unroll
        for (int t = 0; t < kPfTiles; ++t) {
          if (n_s > 0 && !mbar_wait(&s_free[t], (uint32_t)((n_s - 1) & 1), &abort_flag))
            return false;
          tc_fence_after();
          issue_qk(t, k_addr);
        }
        ++n_s;
        if (last_of_item) tc_commit(q_empty);
        tc_commit(&ring_empty[slot]);
        next_slot();
        return true;
      };

      // The items with a key tile, in this CTA's order, as their key-tile
      // count (0: none left) and whether their last V tile has its tail
      // zeroed.  The next one is decoded once the current one's first S pair
      // is out, so the divisions stay off the issue path between two items.
      int r_next = 0;
      auto find_next = [&](int& n_kv_out, bool& tail_out) {
        n_kv_out = 0;
        tail_out = false;
        for (;; ++r_next) {
          const int w = prefill_item_index(r_next, cta, G);
          if (w >= p.n_items) return;
          const PrefillItem it = prefill_item<kPaged>(p, w);
          if (it.n_kv > 0) {
            n_kv_out = it.n_kv;
            tail_out = it.v_tail_fill;
            ++r_next;
            return;
          }
        }
      };
      int n_kv, n_kv_next;
      bool tail, tail_next;
      find_next(n_kv, tail);
      while (ok && n_kv > 0) {
        ok = mbar_wait(q_full, (uint32_t)(n_done & 1), &abort_flag);
        if (ok) ok = issue_s(n_kv == 1);
        find_next(n_kv_next, tail_next);
        for (int j = 0; j < n_kv && ok; ++j) {
          if (j + 1 < n_kv) {
            ok = issue_s(j + 2 == n_kv);
            if (!ok) break;
          }
          // O_X += P_X(j).V_j as soon as P_X(j) is in shared memory
          ok = mbar_wait(&ring_full[slot], phase, &abort_flag);
          if (ok && tail && j == n_kv - 1) {
            ok = mbar_wait(v_tail, (uint32_t)(n_vt & 1), &abort_flag);
            ++n_vt;
          }
          if (!ok) break;
          const uint32_t v_addr = ring_addr + slot * L::kTileBytes;
#pragma unroll
          for (int t = 0; t < kPfTiles; ++t) {
            ok = mbar_wait(&p_full[t], (uint32_t)(n_pv & 1), &abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_pv(t, v_addr, j > 0);
          }
          if (!ok) break;
          ++n_pv;
          tc_commit(&ring_empty[slot]);
          next_slot();
        }
        ++n_done;
        n_kv = n_kv_next;
        tail = tail_next;
      }
      // every MMA of this thread must finish before tensor memory is freed
      tc_commit(mma_drain);
      mbar_wait(mma_drain, 0, nullptr);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPfRegsSoftmax));
    // ======================================================== softmax
    const int t = (warp >> 2) - 1;                // query tile of this warpgroup
    const int quarter = warp & 3;                 // TMEM lane quarter of this warp
    const int r_row = quarter * 32 + lane;        // row within the tile
    const bool store_thread = quarter == 0 && lane == 0;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_addr = lane_addr + L::col_s(t);
    const uint32_t o_addr = lane_addr + L::col_o(t);
    uint8_t* sp_t = sp + t * L::kPBytes;          // P_t; O_t is staged here for its store
    const uint32_t row_addr = smem_u32(sp_t) + r_row * 128;   // this row of P_t (and of O_t)
    const uint32_t sw = (uint32_t)(r_row & 7);     // its 128-byte swizzle
    int n_step = 0;   // S_t read and P_t written so far, over all items (s_full and
                      // pv_done phases)
    bool ok = true;

    for (int r = 0;; ++r) {
      const int w = prefill_item_index(r, cta, G);
      if (w >= p.n_items) break;
      // the loop needs only the key-tile count and the last key this row
      // sees (bottom-right causal, sequence end); the epilogue decodes the
      // item again rather than keep it live
      int n_kv, kmax;
      {
        const PrefillItem it = prefill_item<kPaged>(p, w);
        n_kv = it.n_kv;
        kmax = it.skv_b - 1;
        if (p.causal)
          kmax = (int)min((long long)it.q_blk + t * it.dr + r_row + it.off, (long long)kmax);
      }
      float m_ref = -INFINITY;  // exponent reference (log2 domain)
      float l_sum = 0.f;        // sum of the bf16-rounded weights that feed P.V (normalises O)
      float l_exact = 0.f;      // sum of the unrounded weights (gives the LSE)
      // P_t's slot still holds the previous item's O until its store has
      // read it: the storing thread waits for that, then the warpgroup meets
      // (all of it: the previous item ended with every thread together)
      if (r > 0) {
        if (store_thread) tma_store_wait_read();
        bar_sync_or(3 + t, 128, false);
      }

      for (int j = 0; j < n_kv && ok; ++j) {
        ok = mbar_wait_warp(&s_full[t], (uint32_t)(n_step & 1), &abort_flag);
        if (!ok) break;
        tc_fence_after();
        float s[kPfBN];
        {
          uint32_t* su = reinterpret_cast<uint32_t*>(s);
#pragma unroll
          for (int c = 0; c < kPfBN; c += 32) tmem_ld32(s_addr + c, su + c);
          tc_wait_ld();
        }
        // S_t is in registers: the MMA warp may overwrite it with the next S_t
        tc_fence_before();
        mbar_arrive(&s_free[t]);
        const int kv0 = j * kPfBN;
        if (__any_sync(0xffffffffu, kv0 + kPfBN - 1 > kmax)) {   // a key hidden from a row
          const int cmax = kmax - kv0;
#pragma unroll
          for (int c = 0; c < kPfBN; ++c) s[c] = (c <= cmax) ? s[c] : -INFINITY;
        }
        // row max: four independent three-input chains
        float mx;
        {
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < kPfBN; c += 8) {
            m0 = max3f(m0, s[c], s[c + 1]);
            m1 = max3f(m1, s[c + 2], s[c + 3]);
            m2 = max3f(m2, s[c + 4], s[c + 5]);
            m3 = max3f(m3, s[c + 6], s[c + 7]);
          }
          mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
        }
        const float m_tile = mx * p.scale_log2;
        // move the reference only when the max grew by more than the threshold
        const bool move = m_tile > m_ref + kPfRescaleThreshold;
        float alpha = 1.f;
        if (move) {
          alpha = fast_exp2(m_ref - m_tile);   // 0 when m_ref = -inf
          m_ref = m_tile;
          l_sum *= alpha;
          l_exact *= alpha;
        }
        if (j > 0) {
          // PV_t(j-1) must be done before O_t is rescaled or P_t is overwritten
          ok = mbar_wait_warp(&pv_done[t], (uint32_t)((n_step - 1) & 1), &abort_flag);
          if (!ok) break;
          tc_fence_after();
        }
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // Rescale O_t in TMEM (PV_t(j) is not issued before P_t(j) is ready)
          // (16 columns at a time: S is live in registers here)
#pragma unroll
          for (int c = 0; c < D; c += 16) {
            uint32_t ov[16];
            tmem_ld16(o_addr + c, ov);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st16(o_addr + c, ov);
          }
        }
        // P = exp2(s * scale_log2 - m_ref), rounded to bf16 and stored to
        // shared memory chunk by chunk (K-major, 128-byte swizzled: the
        // layout of the A operand of the P.V MMA).  O is normalised by the
        // sum of the same rounded weights, so it stays a convex combination
        // of V rows even when the lazy reference leaves weights above 1; the
        // LSE uses the exact sum.
        const float neg_ref = (m_ref == -INFINITY) ? 0.f : -m_ref;
        {
          const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t ref2 = f2_pack(neg_ref, neg_ref);
          uint64_t es0 = 0, es1 = 0;   // exact partial sums, packed (0.0f pairs)
          float rs0 = 0.f, rs1 = 0.f, rs2 = 0.f, rs3 = 0.f;   // rounded partial sums
#pragma unroll
          for (int c8 = 0; c8 < kPfBN; c8 += 8) {
            uint32_t wv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = c8 + 2 * q;
              float x0, x1, e0, e1;
              f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), scale2, ref2), x0, x1);
              e0 = fast_exp2(x0);
              e1 = fast_exp2(x1);
              wv[q] = pack_bf16x2(e0, e1);
              // the rounded weights are added straight from their bf16 halves
              if (q & 1) {
                es1 = f2_add(es1, f2_pack(e0, e1));
                add_bf16x2_to_f32(rs2, rs3, wv[q]);
              } else {
                es0 = f2_add(es0, f2_pack(e0, e1));
                add_bf16x2_to_f32(rs0, rs1, wv[q]);
              }
            }
            const int chunk = c8 >> 3, h = chunk >> 3, ch = chunk & 7;
            st_shared_v4(row_addr + h * L::kHalfBytes + ((ch ^ sw) << 4), wv[0], wv[1], wv[2],
                         wv[3]);
          }
          float c2, d2;
          f2_unpack(f2_add(es0, es1), c2, d2);
          l_sum += (rs0 + rs1) + (rs2 + rs3);
          l_exact += c2 + d2;
        }
        tc_wait_st();   // O rescale stores, if any, before PV_t(j) may run
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
        ++n_step;
      }

      // ---- epilogue (the item is decoded again while the last P.V runs)
      const PrefillItem it =
          prefill_item<kPaged>(p, prefill_item_index(opaque_int(r), cta, G));
      const int q0 = it.q_blk + t * it.dr;          // first query row of the tile
      const int hq = it.hq0 + t * it.dh;            // query head of the tile
      const int qi = q0 + r_row;                    // query index
      if (ok && n_kv > 0)
        ok = mbar_wait_warp(&pv_done[t], (uint32_t)((n_step - 1) & 1), &abort_flag);
      if (ok) {
        tc_fence_after();
        // a row that never saw a visible key (m_ref = -inf) gets o = 0 and
        // lse = -inf (its sum may only hold the clamped 2^-125 of masked
        // keys); rows of the padding past this sequence's chunk get o = 0
        const bool any_key = m_ref != -INFINITY && qi < it.sq_b;
        const float inv_l = (any_key && l_sum > 0.f) ? 1.f / l_sum : 0.f;
        // O tile -> bf16 -> shared memory (P_t's slot: the last P.V is done
        // with it) in the 128-byte swizzled layout of the O tensor map
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t ov[32];
          if (it.n_kv > 0) {
            tmem_ld32(o_addr + c, ov);
            tc_wait_ld();
          }
          if (it.n_kv == 0 || !any_key) {   // (padding rows may hold NaN from padded queries)
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0u;
          }
          const int h = c / 64;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {          // 4 chunks of 8 columns
            const int chunk = ((c % 64) / 8) + ch;
            const float* f = reinterpret_cast<const float*>(ov + ch * 8);
            st_shared_v4(row_addr + h * L::kHalfBytes + ((chunk ^ sw) << 4),
                         pack_bf16x2(f[0] * inv_l, f[1] * inv_l),
                         pack_bf16x2(f[2] * inv_l, f[3] * inv_l),
                         pack_bf16x2(f[4] * inv_l, f[5] * inv_l),
                         pack_bf16x2(f[6] * inv_l, f[7] * inv_l));
          }
        }
        if (p.lse != nullptr && qi < p.Sq) {   // padding rows get -inf
          const float lse2 = (any_key && l_exact > 0.f) ? m_ref + fast_log2(l_exact) : -INFINITY;
          p.lse[((size_t)it.b * p.Hq + hq) * p.Sq + qi] = lse2 * 0.69314718055994530942f;
        }
        fence_proxy_async_smem();
        tc_fence_before();   // O_t read before the next item's first P.V overwrites it
      }
      // the four warps of this tile meet here whatever happened; store only
      // if none of the CTA's warps gave up, else stop
      const bool stop = bar_sync_or(1 + t, 128, !ok || abort_flag);
      if (stop) break;
      if (store_thread && q0 < p.Sq) {
#pragma unroll
        for (int h = 0; h < kHalves; ++h)
          tma_store_4d(&tm_o, sp_t + h * L::kHalfBytes, h * 64, q0, hq, it.b);
        tma_store_commit();
      }
    }
    if (store_thread) tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace frt
