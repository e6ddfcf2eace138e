// prefill_sm100.cuh -- tiled causal/non-causal attention forward on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes is the FlashAttention-style forward of the "Real-time
// inference optimisation" page (llmapi-app.pages.dev), section "Flash
// Attention optimisation": for each 128-query tile, loop over 128-key tiles,
// S = Q.K^T, online softmax (running max and sum, accumulator rescaled when
// the max moves), O += P.V, finally O / l; plus causal masking and MQA/GQA
// from the "FlashRT-HF-kernels" page (zingnex.cn), section "Attention
// optimisation".  Key tiles that the causal mask hides completely are never
// loaded or multiplied.
//
// Roles (one CTA = one 128-query tile of one query head, 6 warps):
//   warp 0    TMA producer: Q once, then K and V tiles into a ring of
//             shared-memory slots in the order the MMA warp consumes them
//             (K0, K1, V0, K2, V1, ...), 128-byte swizzled.
//   warp 1    allocates tensor memory and issues the MMAs from one thread:
//             S_j = Q.K_j^T into one of two S buffers (TMEM, fp32), then
//             O += P_j.V_j with P_j read from TMEM (it overwrites S_j as
//             bf16) and O accumulating in TMEM.
//   warps 2-5 softmax: each thread owns one query row (= one TMEM lane);
//             it reads its S row, masks, keeps the running max and sum in
//             the exp2 domain (scale*log2(e) folded in), writes P back to
//             TMEM and rescales O in TMEM when needed; then the epilogue
//             (O / l -> bf16 -> shared memory -> TMA store, and the LSE).
// Rescaling is lazy: the exponent reference only moves when the row max
// grows by more than 2^8, so O is rarely touched; the result is exact either
// way because numerator and denominator share the reference.
#pragma once

#include "frt_device.cuh"

namespace frt {

constexpr int kPfBM = 128;             // query rows per tile (TMEM lanes)
constexpr int kPfBN = 128;             // keys per tile
constexpr int kPfThreads = 192;
constexpr float kPfRescaleThreshold = 8.0f;   // log2 units

template <int D>
struct PrefillSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = 128 * 128;              // 128 rows x 64 bf16
  static constexpr int kTileBytes = kHalves * kHalfBytes;   // Q, K or V tile
  // K/V ring; D=64 keeps 8 slots so that one CTA fills the SM (the kernel
  // allocates all 512 TMEM columns, so a second resident CTA would only wait)
  static constexpr int kSlots = (D == 128) ? 4 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kTileBytes;
  static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 2 + 2 + 1;
  static constexpr int kBytes = 1024 + kBarOff + kNumBars * 8 + 64;
  // TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
};

struct PrefillParams {
  float* lse;          // [B, Hq, Sq] or nullptr
  __nv_bfloat16* o;    // [B, Hq, Sq, D] (used only to zero rows without keys)
  int B, Hq, Hkv, g, Sq, Skv, causal, n_qtiles;
  float scale_log2;
};

template <int D>
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
  uint8_t* ring = smem + L::kRingOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* ring_full = bars + 1;
  uint64_t* ring_empty = ring_full + kSlots;
  uint64_t* s_full = ring_empty + kSlots;     // [2]
  uint64_t* p_full = s_full + 2;              // [2]
  // pv_done[b]: PV_j with j % 2 == b completed.  One barrier per S buffer, so
  // that a waiter never falls two phases behind (a parity wait on a barrier
  // that completed twice since would return at once).
  uint64_t* pv_done = p_full + 2;             // [2]
  uint64_t* mma_drain = pv_done + 2;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- tile coordinates (heaviest causal tiles are scheduled first)
  const int bh = blockIdx.x;                 // b * Hq + hq
  const int qt = p.causal ? (p.n_qtiles - 1 - (int)blockIdx.y) : (int)blockIdx.y;
  const int b = bh / p.Hq, hq = bh % p.Hq;
  const int kv_row = b * p.Hkv + hq / p.g;   // z coordinate in the K/V maps
  const int q0 = qt * kPfBM;
  const int off = p.Skv - p.Sq;              // bottom-right causal alignment
  const int q_last = min(q0 + kPfBM - 1, p.Sq - 1);
  const int n_kv_all = (p.Skv + kPfBN - 1) / kPfBN;
  int n_kv = n_kv_all;
  if (p.causal) {
    const int lim = q_last + off;            // largest key any row of the tile sees
    n_kv = lim < 0 ? 0 : min(n_kv_all, lim / kPfBN + 1);
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(mma_drain, 1);
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

  if (warp == 0) {
    // ================================================= TMA producer
    if (lane == 0 && n_kv > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(q_full, L::kTileBytes);
#pragma unroll
      for (int h = 0; h < kHalves; ++h)
        tma_load_3d(sq + h * L::kHalfBytes, &tm_q, q_full, h * 64, q0, bh);
      int slot = 0;
      uint32_t phase = 0;
      auto load = [&](const CUtensorMap* tm, int j) -> bool {
        if (!mbar_wait(&ring_empty[slot], phase ^ 1u, &abort_flag)) return false;
        mbar_arrive_expect_tx(&ring_full[slot], L::kTileBytes);
        uint8_t* dst = ring + slot * L::kTileBytes;
#pragma unroll
        for (int h = 0; h < kHalves; ++h)
          tma_load_3d(dst + h * L::kHalfBytes, tm, &ring_full[slot], h * 64, j * kPfBN, kv_row);
        if (++slot == kSlots) { slot = 0; phase ^= 1u; }
        return true;
      };
      // the MMA warp consumes K0, then for each j: K_{j+1} (if any), V_j
      bool ok = load(&tm_k, 0);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv) ok = load(&tm_k, j + 1);
        if (ok) ok = load(&tm_v, j);
      }
      if (!ok) __nanosleep(100000);
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kPfBM, kPfBN, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(kPfBM, D, false, true);
      const uint32_t sq_addr = smem_u32(sq);
      const uint32_t ring_addr = smem_u32(ring);
      int slot = 0;
      uint32_t phase = 0;
      bool ok = mbar_wait(q_full, 0, &abort_flag);

      auto issue_qk = [&](int sbuf) {
        const uint32_t k_addr = ring_addr + slot * L::kTileBytes;
        const uint32_t d_tmem = tmem + (sbuf ? L::kColS1 : L::kColS0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks >> 2) * L::kHalfBytes + (ks & 3) * 32;
          tc_mma_ss(d_tmem, umma_desc_sw128(sq_addr + koff, 16, 1024),
                    umma_desc_sw128(k_addr + koff, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sbuf]);
        tc_commit(&ring_empty[slot]);
        if (++slot == kSlots) { slot = 0; phase ^= 1u; }
      };
      auto issue_pv = [&](int sbuf, bool accumulate) {
        const uint32_t v_addr = ring_addr + slot * L::kTileBytes;
        const uint32_t a_tmem = tmem + (sbuf ? L::kColS1 : L::kColS0);
#pragma unroll
        for (int kk = 0; kk < kPfBN / 16; ++kk) {
          tc_mma_ts(tmem + L::kColO, a_tmem + kk * 8,
                    umma_desc_sw128(v_addr + kk * 2048, L::kHalfBytes, 1024), idesc_pv,
                    (accumulate || kk > 0) ? 1u : 0u);
        }
        tc_commit(&pv_done[sbuf]);
        tc_commit(&ring_empty[slot]);
        if (++slot == kSlots) { slot = 0; phase ^= 1u; }
      };

      if (ok) ok = mbar_wait(&ring_full[slot], phase, &abort_flag);
      if (ok) {
        tc_fence_after();
        issue_qk(0);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv) {
          ok = mbar_wait(&ring_full[slot], phase, &abort_flag);
          // S buffer (j+1)%2 still holds P_{j-1} until PV_{j-1} completes
          if (ok && j >= 1)
            ok = mbar_wait(&pv_done[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), &abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_qk((j + 1) & 1);
        }
        ok = mbar_wait(&p_full[j & 1], (uint32_t)((j >> 1) & 1), &abort_flag);
        if (ok) ok = mbar_wait(&ring_full[slot], phase, &abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(j & 1, j > 0);
      }
      // every MMA of this thread must finish before tensor memory is freed
      tc_commit(mma_drain);
      mbar_wait(mma_drain, 0, nullptr);
    }
  } else {
    // ======================================================== softmax
    const int quarter = warp & 3;                 // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;            // row within the tile
    const int qi = q0 + r;                        // query index
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const long long row_lim = p.causal ? (long long)qi + off : (long long)1 << 40;
    float m_ref = -INFINITY;                      // exponent reference (log2 domain)
    float l_sum = 0.f;      // sum of the bf16-rounded weights that feed P.V (normalises O)
    float l_exact = 0.f;    // sum of the unrounded weights (gives the LSE)
    bool ok = true;

    for (int j = 0; j < n_kv && ok; ++j) {
      ok = mbar_wait_warp(&s_full[j & 1], (uint32_t)((j >> 1) & 1), &abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_addr = lane_addr + ((j & 1) ? L::kColS1 : L::kColS0);
      float s[kPfBN];
      {
        uint32_t* su = reinterpret_cast<uint32_t*>(s);
#pragma unroll
        for (int c = 0; c < kPfBN; c += 32) tmem_ld32(s_addr + c, su + c);
        tc_wait_ld();
      }
      const int kv0 = j * kPfBN;
      const bool need_mask = (p.causal && kv0 + kPfBN - 1 > q0 + off) || (kv0 + kPfBN > p.Skv);
      if (need_mask) {
        long long cmax = row_lim - kv0;
        const long long tail = (long long)p.Skv - 1 - kv0;
        if (tail < cmax) cmax = tail;
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
      if (j > 0 && __any_sync(0xffffffffu, move)) {
        // rescale O (TMEM) once PV_{j-1} has landed
        ok = mbar_wait_warp(&pv_done[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), &abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t ov[32];
          tmem_ld32(lane_addr + L::kColO + c, ov);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(lane_addr + L::kColO + c, ov);
        }
      }
      // P = exp2(s * scale_log2 - m_ref), rounded to bf16, written over S
      const float neg_ref = (m_ref == -INFINITY) ? 0.f : -m_ref;
      uint32_t pk[kPfBN / 2];
      {
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t ref2 = f2_pack(neg_ref, neg_ref);
        uint64_t rs0 = 0, rs1 = 0, es0 = 0, es1 = 0;   // packed partial sums (0.0f pairs)
#pragma unroll
        for (int c = 0; c < kPfBN; c += 2) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), scale2, ref2), x0, x1);
          const float e0 = fast_exp2(x0), e1 = fast_exp2(x1);
          const uint32_t w = pack_bf16x2(e0, e1);
          pk[c / 2] = w;
          // O is normalised by the same rounded weights that feed P.V, so that
          // it stays a convex combination of V rows; the LSE uses the exact sum
          const uint64_t wr = f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
          const uint64_t we = f2_pack(e0, e1);
          if ((c & 2) == 0) { rs0 = f2_add(rs0, wr); es0 = f2_add(es0, we); }
          else              { rs1 = f2_add(rs1, wr); es1 = f2_add(es1, we); }
        }
        float a, b2, c2, d2;
        f2_unpack(f2_add(rs0, rs1), a, b2);
        f2_unpack(f2_add(es0, es1), c2, d2);
        l_sum += a + b2;
        l_exact += c2 + d2;
      }
      tmem_st32(s_addr, pk);
      tmem_st32(s_addr + 32, pk + 32);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }

    // ---- epilogue
    if (ok && n_kv > 0)
      ok = mbar_wait_warp(&pv_done[(n_kv - 1) & 1], (uint32_t)(((n_kv - 1) >> 1) & 1), &abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv_l = (l_sum > 0.f) ? 1.f / l_sum : 0.f;
      // O tile -> bf16 -> shared memory (the Q slot, free now) in the
      // 128-byte swizzled layout of the O tensor map
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t ov[32];
        if (n_kv > 0) {
          tmem_ld32(lane_addr + L::kColO + c, ov);
          tc_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0u;
        }
        const int h = c / 64;
        uint8_t* row_base = sq + h * L::kHalfBytes + r * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {          // 4 chunks of 8 columns
          const int chunk = ((c % 64) / 8) + ch;
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(ov[ch * 8 + 0]) * inv_l,
                            __uint_as_float(ov[ch * 8 + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(ov[ch * 8 + 2]) * inv_l,
                            __uint_as_float(ov[ch * 8 + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(ov[ch * 8 + 4]) * inv_l,
                            __uint_as_float(ov[ch * 8 + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(ov[ch * 8 + 6]) * inv_l,
                            __uint_as_float(ov[ch * 8 + 7]) * inv_l);
          *reinterpret_cast<uint4*>(row_base + ((chunk ^ (r & 7)) << 4)) = v;
        }
      }
      if (p.lse != nullptr && qi < p.Sq) {
        const float lse2 = (l_exact > 0.f) ? m_ref + fast_log2(l_exact) : -INFINITY;
        p.lse[(size_t)bh * p.Sq + qi] = lse2 * 0.69314718055994530942f;
      }
      fence_proxy_async_smem();
    }
    // all four softmax warps meet here whatever happened; store only if none gave up
    const bool stop = bar_sync_or(1, 128, !ok || abort_flag);
    if (!stop && warp == 2 && lane == 0) {
#pragma unroll
      for (int h = 0; h < kHalves; ++h) tma_store_3d(&tm_o, sq + h * L::kHalfBytes, h * 64, q0, bh);
      tma_store_commit();
      tma_store_wait_all();
    }
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
