// decode_splitkv.cuh -- split-KV decode attention (one query token per
// sequence) over a paged or contiguous KV cache, for sm_100a.
//
// What it computes: softmax attention of each query head over its sequence's
// cached keys, as the online-softmax kernel of the "Real-time inference
// optimisation" page (llmapi-app.pages.dev, section "Flash Attention
// optimisation") does, over a KV cache cut into 16-token pages (same page,
// method paged_attention), with MQA/GQA head sharing ("FlashRT-HF-kernels"
// page, section "Attention optimisation").  Partial results over disjoint
// key ranges are combined by their log-sum-exp, the correct form of that
// page's per-page sum.
//
// Work plan (flattened split-KV).  A segment is (sequence b, KV head kvh,
// group of up to 16 query heads of that KV head); it owns ceil(len_b/16)
// pages.  All segments' pages are laid end to end (units) and the CTAs of the
// grid take equal contiguous shares of that line, so every CTA streams the
// same number of pages whatever the length mix.  The piece of a segment that
// falls inside one CTA is reduced to one partial (o, lse); a segment wholly
// inside one CTA is written out directly.  The partials of split segments
// are combined by log-sum-exp in a second, small kernel (decode_merge_kernel)
// that spreads every (sequence, query head) row over its own CTA; it is
// launched as a programmatic dependent, so it is resident and waiting when
// the streaming kernel ends.  No CTA ever waits for another.
//
// Inside a CTA (two per SM; three for the FP8 cache with one head tile):
// warp 0 streams pages into a ring of
// shared-memory stages with TMA (one 128-byte swizzled box per page and
// matrix, one mbarrier per stage), looking pages up in the block table;
// warps 1..W (DecodeCfg) each take one or two pages of every stage and compute
// S^T = K.Q^T and O^T += V^T.P^T with warp-level MMAs (bf16, or f16 from an
// e4m3 cache) in which a page's
// tokens form the M dimension of the first and the segment's query heads the
// N dimension of both, so each K/V page is read from HBM once for all heads
// of its group.  Scores live in the exp2 domain (scale * log2(e) folded in).
// At the end of a piece the warps' states are combined in registers (through
// shared memory) and written by one warp.
//
// Cluster mode (kCluster, contiguous cache only): no workspace and no second
// kernel.  Each segment is owned by one thread-block cluster of C <= 16 CTAs;
// CTA r of the cluster streams pages [r*n/C, (r+1)*n/C) of the segment's n
// pages, leaves its state (unnormalised output, running max and both sums)
// in its own shared memory, and after a cluster barrier the cluster's
// threads merge the C states by log-sum-exp, reading the other CTAs' shared
// memory directly (distributed shared memory), and write the final rows.
#pragma once

#include "frt_device.cuh"

namespace frt {

constexpr int kDecPage = 16;          // tokens per page (one MMA K-step)
// Consumer warps per CTA (a power of two) and the pages each takes per
// stage.  With one 8-head tile the consumers, not HBM, set the pace with two
// warps, so there are four of one page each (a stage of 4 pages: 32 KB for
// bf16, 16 KB for FP8).  Otherwise two warps of two pages.
// CTAs per SM and ring size: the FP8 cache with one head tile is
// consumer-latency-bound, so its SMs take three CTAs of a 48 KB ring (the
// kernel fits in 122 registers) instead of two of 96 KB; measured on B200:
// 256k decode 52.5 -> 51.4 us, the paged B4 one unchanged.
template <bool kFp8, int kHT>
struct DecodeCfg {
  static constexpr int kWarps = (kHT == 1) ? 4 : 2;
  static constexpr int kPagesPerWarp = (kHT == 1) ? 1 : 2;
  static constexpr int kStagePages = kWarps * kPagesPerWarp;
  static constexpr int kThreads = 32 * (kWarps + 1);
  static constexpr int kCtasPerSm = (kFp8 && kHT == 1) ? 3 : 2;
  static constexpr int kRingBytes = (kFp8 && kHT == 1 ? 48 : 96) * 1024;
};
// bf16 cache: up to two CTAs share an SM: two independent TMA rings per SM
// keep more page copies in flight than one ring twice as deep.  The default
// grid aims at about 18 MiB of page copies in flight over the whole GPU (192
// CTAs of a 96 KB ring); measured on B200, fewer starve HBM of requests and
// more (two rings on every SM, 28 MiB) read measurably slower.
constexpr int kDecCtasPerSm = 2;
constexpr long long kDecInFlightBytes = 18ll << 20;
constexpr int kDecHeadsPerSeg = 16;   // MMA M dimension
// The producer reads block-table entries for 32 pages at a time (one per
// lane) and hands them out stage by stage, so a stage must divide 32 pages.
static_assert(32 % DecodeCfg<false, 1>::kStagePages == 0 && 32 % DecodeCfg<false, 2>::kStagePages == 0 &&
                  32 % DecodeCfg<true, 1>::kStagePages == 0 && 32 % DecodeCfg<true, 2>::kStagePages == 0,
              "stages of whole windows");
constexpr int kDecMaxBatch = 1024;    // prefix table held in shared memory

struct DecodeParams {
  const __nv_bfloat16* q;        // [B, Hq, D]
  __nv_bfloat16* o;              // [B, Hq, D]
  float* lse;                    // [B, Hq] natural log, or nullptr
  const int32_t* block_table;    // paged: [B, max_pages]; contiguous: nullptr
  const int32_t* seq_lens;       // paged: [B] (device); contiguous: nullptr
  int max_pages;                 // paged: block-table row length
  int num_pages;                 // paged: physical pages; entries outside [0, num_pages)
                                 // are read from row `bad_row` (past the end: zeros)
  int bad_row;                   // rows of the [rows, D] view of the cache (< 2^31)
  int contig_len;                // contiguous: keys per sequence (Skv)
  int B, Hq, Hkv, g, hgroups;    // g = Hq / Hkv, hgroups = ceil(g / 16)
  int parts;                     // CTAs of the streaming kernel's grid
  float scale_log2;              // scale * log2(e)
  const float* k_scale;          // FP8 cache: [Hkv] value = code * k_scale[h]; else nullptr
  const float* v_scale;          // FP8 cache: [Hkv]; else nullptr
  float* ws_o;                   // [slots, 16, D] fp32 partial outputs (normalised)
  float* ws_lse;                 // [slots, 16] fp32 partial LSE (log2 domain)
  int2* ws_seg;                  // [segments] CTAs holding its pieces {first, last};
                                 // {-1, -1}: written out whole (or empty)
};

// kFp8: the cache holds FP8 e4m3 codes (one byte per element, D = 128 only):
// a page is one 16 x 128-byte box; otherwise bf16 pages of D/64 boxes of
// 16 rows x 64 elements.
template <int D, bool kFp8 = false, int kHT = 2>
struct DecodeSmem {
  static_assert(!kFp8 || D == 128, "the FP8 cache is supported at D = 128");
  using Cfg = DecodeCfg<kFp8, kHT>;
  static constexpr int kHalves = D / 64;
  static constexpr int kBoxBytes = kDecPage * 128;                    // 16 rows x 128 bytes
  static constexpr int kPageBytes = kDecPage * D * (kFp8 ? 1 : 2);   // K or V of one page
  static constexpr int kStageBytes = Cfg::kStagePages * 2 * kPageBytes; // K+V of a stage
  static constexpr int kStages = Cfg::kRingBytes / kStageBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  // cross-warp combine: one warp's register state in fragment order
  // (D/16 m-tiles x kHT head tiles x 4 accumulators, then m, l, l_exact for
  // 2 heads of each head tile)
  static constexpr int kFragFloats = (D / 16) * kHT * 4 + 6 * kHT;
  static constexpr int kScratchFloats = (Cfg::kWarps / 2) * kFragFloats * 32;
  // cluster mode: a CTA's final state reuses the scratch area: unnormalised
  // o of up to 8 * kHT heads, then per head {running max, sum of the rounded
  // weights, exact sum, unused} (one 16-byte load)
  static constexpr int kXchO = 0;
  static constexpr int kXchS = kHT * 8 * D;
  static_assert(kXchS + kHT * 8 * 4 <= kScratchFloats, "cluster exchange fits in the scratch area");
  static constexpr int kScratchOff = kRingBytes;
  static constexpr int kPrefixOff = kScratchOff + kScratchFloats * 4;
  static constexpr int kBarOff = kPrefixOff + ((kDecMaxBatch + 1) * 4 + 15) / 16 * 16;
  static constexpr int kBytes = 1024 /*alignment slack*/ + kBarOff + 2 * kStages * 8;
  static_assert(kBarOff % 8 == 0, "mbarriers need 8-byte alignment");
  // per SM: 228 KB, of which each CTA also reserves 1 KB (static shared
  // variables live in the slack below)
  static_assert(Cfg::kCtasPerSm * (kBytes + 1024 + 64) <= 228 * 1024, "shared memory budget");
};

// Pages of sequence b (seq_len clamped to [0, max_pages * 16]).
__device__ __forceinline__ int dec_pages_of(const DecodeParams& p, int b) {
  if (p.seq_lens == nullptr) return (p.contig_len + kDecPage - 1) / kDecPage;
  int len = p.seq_lens[b];
  len = len < 0 ? 0 : len;
  long long cap = (long long)p.max_pages * kDecPage;
  if (len > cap) len = (int)cap;
  return (len + kDecPage - 1) / kDecPage;
}

__device__ __forceinline__ int dec_len_of(const DecodeParams& p, int b) {
  if (p.seq_lens == nullptr) return p.contig_len;
  int len = p.seq_lens[b];
  len = len < 0 ? 0 : len;
  long long cap = (long long)p.max_pages * kDecPage;
  return len > cap ? (int)cap : len;
}

// CTA whose share of the unit line [0, T) holds unit u (shares are
// [floor(c*T/C), floor((c+1)*T/C)); requires T >= C so none is empty).
__device__ __forceinline__ int dec_cta_of(long long u, long long T, int C) {
  return (int)(((u + 1) * (long long)C - 1) / T);
}

// Swizzled shared-memory address of the 16-byte chunk holding element
// (row, col) of a 16 x 64 bf16 TMA box written with 128-byte swizzling.
__device__ __forceinline__ uint32_t sw128_addr(uint32_t box_base, int row, int col) {
  return box_base + row * 128 + ((((col >> 3) ^ (row & 7))) << 4);
}

// Byte address in a 16 x 128-byte page box written with 128-byte swizzling
// of the 16-byte chunk `chunk` of row `row`.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t box_base, int row, int chunk) {
  return box_base + row * 128 + (((chunk ^ (row & 7))) << 4);
}

// kHT: 8-head tiles per segment (1 when a KV head serves at most 8 query
// heads, else 2; a segment holds at most 16 query heads).
// kFp8: K/V pages hold e4m3 codes with per-KV-head scales.  The codes become
// f16 in registers (exact) and the MMAs run in f16; K's scale is folded into
// the score scale and V's into the final normalisation.  A page's K rows are
// loaded by ldmatrix as byte quadruples, so the MMA's k index walks d in the
// order (4c, 4c+1 | 4c+2, 4c+3) per 16-d step, and Q's fragments follow the
// same order; V^T's rows come out as the even and odd d of each pair.
// kCluster: cluster mode (see the top of this file): contiguous bf16 cache,
// launched with a cluster of C CTAs per segment; nothing goes to a workspace.
template <int D, int kHT, bool kFp8, bool kCluster = false>
__global__ void __launch_bounds__(DecodeCfg<kFp8, kHT>::kThreads, DecodeCfg<kFp8, kHT>::kCtasPerSm)
decode_splitkv_kernel(const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  static_assert(!(kCluster && kFp8), "cluster mode reads a bf16 cache");
  using L = DecodeSmem<D, kFp8, kHT>;
  constexpr int kDecWarps = DecodeCfg<kFp8, kHT>::kWarps;            // consumer warps
  constexpr int kDecStagePages = DecodeCfg<kFp8, kHT>::kStagePages;
  constexpr int kPPW = DecodeCfg<kFp8, kHT>::kPagesPerWarp;            // pages per warp per stage
  constexpr int kStages = L::kStages;
  constexpr int kKSteps = D / 16;     // MMA K-steps of K.Q^T

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* scratch = reinterpret_cast<float*>(smem + L::kScratchOff);
  int* prefix = reinterpret_cast<int*>(smem + L::kPrefixOff);   // [B+1] page prefix
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty_bar = full_bar + kStages;
  __shared__ int abort_flag;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int nseg_b = p.Hkv * p.hgroups;   // segments per sequence

  // Inputs may come from the kernel before this one in the stream: wait for
  // it (a no-op unless launched as a programmatic dependent), then let the
  // merge kernel that follows get resident.
  griddep_wait();
  griddep_launch_dependents();

  // ---- per-sequence page prefix (warp 0: chunked scan; not needed in
  // cluster mode, where every sequence has contig_len keys), barriers
  if (warp == 0) {
    const int per = kCluster ? 0 : (p.B + 31) / 32;
    const int b0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (b0 + i < p.B) local += dec_pages_of(p, b0 + i);
    int incl = local;
    for (int off = 1; off < 32; off <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i)
      if (b0 + i < p.B) {
        prefix[b0 + i] = run;
        run += dec_pages_of(p, b0 + i);
      }
    if (!kCluster && lane == 31) prefix[p.B] = incl;
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full_bar[s], 1);
        mbar_init(&empty_bar[s], kDecWarps);
      }
      abort_flag = 0;
      fence_barrier_init();
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
    }
  }
  __syncthreads();

  // unit line (split mode): T units over the C CTAs with a non-empty share
  const long long T = kCluster ? 0 : (long long)prefix[p.B] * nseg_b;
  const int C = kCluster ? 0 : (int)min((long long)gridDim.x, T);
  const int c = blockIdx.x;
  // cluster mode: segment of this cluster, and this CTA's rank among its CTAs
  const int cl_size = kCluster ? (int)cluster_nctarank() : 1;
  const int cl_rank = kCluster ? (int)cluster_ctarank() : 0;
  const int cl_seg = c / cl_size;

  // ---- sequences with no key: o = 0, lse = -inf (spread over the grid)
  for (int b = c; !kCluster && b < p.B; b += gridDim.x) {
    if (prefix[b + 1] != prefix[b]) continue;
    for (int i = threadIdx.x; i < p.Hq * D; i += blockDim.x)
      p.o[(size_t)b * p.Hq * D + i] = __float2bfloat16(0.f);
    if (p.lse != nullptr)
      for (int i = threadIdx.x; i < p.Hq; i += blockDim.x) p.lse[(size_t)b * p.Hq + i] = -INFINITY;
    for (int i = threadIdx.x; i < nseg_b; i += blockDim.x) p.ws_seg[(size_t)b * nseg_b + i] = make_int2(-1, -1);
  }
  if (!kCluster && c >= C) return;

  const long long u_begin = kCluster ? 0 : (long long)c * T / C;
  const long long u_end = kCluster ? 0 : (long long)(c + 1) * T / C;

  // Walk of this CTA's pieces, identical in every warp.  Returns false when
  // the share is exhausted.  (b, seg_in_b) identify the segment, pages
  // [pg0, pg1) of it lie in this CTA, npg = pages of the segment.
  struct Piece {
    int b, seg_in_b, pg0, pg1, npg;
    long long seg_u0;
  };
  auto first_piece = [&](Piece& pc) {
    if constexpr (kCluster) {
      // the cluster's segment; this CTA's equal share of its pages (may be
      // empty when the segment has fewer pages than the cluster has CTAs)
      const int npg = (p.contig_len + kDecPage - 1) / kDecPage;
      pc.b = cl_seg / nseg_b;
      pc.seg_in_b = cl_seg % nseg_b;
      pc.npg = npg;
      pc.seg_u0 = 0;
      pc.pg0 = (int)((long long)cl_rank * npg / cl_size);
      pc.pg1 = (int)((long long)(cl_rank + 1) * npg / cl_size);
      return;
    }
    // largest b with prefix[b] * nseg_b <= u_begin and a non-empty sequence
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if ((long long)prefix[mid] * nseg_b <= u_begin) lo = mid; else hi = mid - 1;
    }
    int b = lo;
    while (prefix[b + 1] == prefix[b]) ++b;   // skip empty sequences
    const int npg = prefix[b + 1] - prefix[b];
    const long long off = u_begin - (long long)prefix[b] * nseg_b;
    pc.b = b;
    pc.seg_in_b = (int)(off / npg);
    pc.npg = npg;
    pc.seg_u0 = (long long)prefix[b] * nseg_b + (long long)pc.seg_in_b * npg;
    pc.pg0 = (int)(off % npg);
    long long seg_end = pc.seg_u0 + npg;
    pc.pg1 = (int)((seg_end < u_end ? seg_end : u_end) - pc.seg_u0);
  };
  auto next_piece = [&](Piece& pc) -> bool {
    if (kCluster) return false;   // one piece per CTA
    long long u = pc.seg_u0 + pc.pg1;
    if (u >= u_end) return false;
    int b = pc.b, s = pc.seg_in_b + 1;
    if (s == nseg_b) {
      s = 0;
      ++b;
      while (prefix[b + 1] == prefix[b]) ++b;
    }
    const int npg = prefix[b + 1] - prefix[b];
    pc.b = b;
    pc.seg_in_b = s;
    pc.npg = npg;
    pc.seg_u0 = u;
    pc.pg0 = 0;
    pc.pg1 = (int)((u + npg < u_end ? u + npg : u_end) - u);
    return true;
  };

  if (warp == 0) {
    // =================================================== producer (TMA)
    int stage = 0;
    uint32_t phase = 0;
    Piece pc;
    first_piece(pc);
    bool ok = true;
    do {
      const int kvh = pc.seg_in_b / p.hgroups;
      // Rows (first token of each page in the [rows, D] view of the cache) of
      // the next 32 pages of this piece, one per lane, so the block table is
      // read in one round trip per 32 pages instead of one per stage and the
      // ring's first stages are issued back to back.
      int win0 = pc.pg0, win_row = 0;
      auto load_window = [&](int first) {
        win0 = first;
        win_row = 0;
        const int page = first + lane;
        if (page < pc.pg1) {
          if (p.block_table != nullptr) {
            // An entry outside [0, num_pages) is never used as an address:
            // the copy starts past the cache's last row, so the page reads as
            // zeros, and the error word records it.  Valid rows are below
            // num_pages * Hkv * 16 < 2^31 (checked by the host).
            const int phys = p.block_table[(size_t)pc.b * p.max_pages + page];
            if ((unsigned)phys < (unsigned)p.num_pages) {
              win_row = (int)(((long long)phys * p.Hkv + kvh) * kDecPage);
            } else {
              win_row = p.bad_row;
              raise_error(kErrBadPage);
            }
          } else {
            win_row = (int)(((long long)pc.b * p.Hkv + kvh) * p.contig_len +
                            (long long)page * kDecPage);
          }
        }
      };
      load_window(pc.pg0);
      for (int pb = pc.pg0; pb < pc.pg1 && ok; pb += kDecStagePages) {
        const int n = min(kDecStagePages, pc.pg1 - pb);
        if (pb + n > win0 + 32) load_window(pb);   // (a stage never straddles two windows)
        const int row = __shfl_sync(0xffffffffu, win_row, (pb - win0 + lane) & 31);
        ok = mbar_wait_warp(&empty_bar[stage], phase ^ 1u, &abort_flag);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(&full_bar[stage], n * 2 * L::kPageBytes);
        __syncwarp();
        if (lane < n) {
          uint8_t* kdst = ring + stage * L::kStageBytes + lane * 2 * L::kPageBytes;
          uint8_t* vdst = kdst + L::kPageBytes;
          if constexpr (kFp8) {
            tma_load_2d(kdst, &tmap_k, &full_bar[stage], 0, row);
            tma_load_2d(vdst, &tmap_v, &full_bar[stage], 0, row);
          } else {
            tma_load_3d(kdst, &tmap_k, &full_bar[stage], 0, row, 0);
            tma_load_3d(vdst, &tmap_v, &full_bar[stage], 0, row, 0);
          }
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    } while (ok && next_piece(pc));
    // Normal exit needs no drain: the consumers wait for every stage issued
    // here before the CTA can finish.  After an abort they may not, so give
    // copies still in flight time to land before this warp leaves.
    if (!ok) __nanosleep(100000);
  } else {

  // ====================================================== consumers (MMA)
  // S^T = K.Q^T with a page's 16 tokens as the MMA M dimension and the
  // segment's query heads as N (8 per head tile), then O^T += V^T.P^T with
  // the head dimension d as M (16 per m-tile), the heads as N and the page's
  // tokens as K.  With a GQA group of 8 no MMA row or column is padding.
  constexpr int kMT = D / 16;            // 16-row m-tiles of d in O^T
  const int cw = warp - 1;               // consumer warp index
  const int r8 = lane >> 2;              // fragment row: token (S^T) or d (O^T), and head of B
  const int qc = lane & 3;               // fragment column pair: heads 2qc, 2qc+1
  const uint32_t ring_u32 = smem_u32(ring);
  constexpr float kLn2 = 0.69314718055994530942f;

  int stage = 0;
  uint32_t phase = 0;
  Piece pc;
  first_piece(pc);
  bool ok = true;
  do {
    const int kvh = pc.seg_in_b / p.hgroups;
    const int hg = pc.seg_in_b % p.hgroups;
    const int h0 = kvh * p.g + hg * kDecHeadsPerSeg;            // first query head
    const int nh = min(kDecHeadsPerSeg, p.g - hg * kDecHeadsPerSeg);
    const int len = dec_len_of(p, pc.b);
    // score scale (exp2 domain) and output scale of this KV head
    const float sl2 = kFp8 ? p.scale_log2 * p.k_scale[kvh] : p.scale_log2;
    const float o_scale = kFp8 ? p.v_scale[kvh] : 1.f;

    // Q^T fragments (B operand of S^T = K.Q^T): head 8*ht + r8, d pairs
    uint32_t qb[kHT][kKSteps][2];
    {
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q + ((size_t)pc.b * p.Hq + h0) * D);
#pragma unroll
      for (int ht = 0; ht < kHT; ++ht) {
        const int head = ht * 8 + r8;
#pragma unroll
        for (int ks = 0; ks < kKSteps; ++ks) {
          if constexpr (kFp8) {
            // d 16ks + 4qc .. +3 as two f16 pairs (the order of the K loads)
            uint2 w = make_uint2(0u, 0u);
            if (head < nh) w = *reinterpret_cast<const uint2*>(q32 + (head * D + ks * 16 + 4 * qc) / 2);
            qb[ht][ks][0] = pack_f16x2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u));
            qb[ht][ks][1] = pack_f16x2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
          } else {
            qb[ht][ks][0] = head < nh ? q32[(head * D + ks * 16 + 2 * qc) / 2] : 0u;
            qb[ht][ks][1] = head < nh ? q32[(head * D + ks * 16 + 8 + 2 * qc) / 2] : 0u;
          }
        }
      }
    }
    // per lane: heads 2qc, 2qc+1 of each head tile (exp2 domain); the sums
    // are this lane's share over its tokens
    float m_run[kHT][2], l_run[kHT][2], le_run[kHT][2];
    float acc[kMT][kHT][4];
#pragma unroll
    for (int ht = 0; ht < kHT; ++ht) {
      m_run[ht][0] = m_run[ht][1] = -INFINITY;
      l_run[ht][0] = l_run[ht][1] = le_run[ht][0] = le_run[ht][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) acc[mt][ht][0] = acc[mt][ht][1] = acc[mt][ht][2] = acc[mt][ht][3] = 0.f;
    }

    for (int pb = pc.pg0; pb < pc.pg1; pb += kDecStagePages) {
      ok = mbar_wait_warp(&full_bar[stage], phase, &abort_flag);
      if (!ok) break;
      const int page_a = pb + kPPW * cw;     // this warp's first page
      int valid[2];
      valid[0] = page_a < pc.pg1 ? min(kDecPage, len - page_a * kDecPage) : 0;
      valid[1] = (kPPW == 2 && page_a + 1 < pc.pg1) ? min(kDecPage, len - (page_a + 1) * kDecPage) : 0;
      if (valid[0] > 0) {
        const int npg = valid[1] > 0 ? 2 : 1;
        const uint32_t base = ring_u32 + stage * L::kStageBytes +
                              kPPW * cw * 2 * L::kPageBytes;
        // ---- S^T = K.Q^T per page (fragment loads of a page issued first)
        float sacc[2][kHT][4];
#pragma unroll
        for (int pg = 0; pg < kPPW; ++pg)
#pragma unroll
          for (int ht = 0; ht < kHT; ++ht) sacc[pg][ht][0] = sacc[pg][ht][1] = sacc[pg][ht][2] = sacc[pg][ht][3] = 0.f;
        {
          const int mi = lane >> 3, j = lane & 7;
          const int tok = (mi & 1) * 8 + j;
#pragma unroll
          for (int pg = 0; pg < kPPW; ++pg) {
            if (pg < npg) {
              const uint32_t kbase = base + pg * 2 * L::kPageBytes;
              if constexpr (kFp8) {
                // matrix mi: tokens (mi&1)*8.., 16-byte chunk 2b + (mi>>1); each
                // ldmatrix covers two K-steps (32 d)
                uint32_t kr[kKSteps / 2][4];
#pragma unroll
                for (int b2 = 0; b2 < kKSteps / 2; ++b2)
                  ldsm_x4(sw128_chunk(kbase, tok, 2 * b2 + (mi >> 1)), kr[b2][0], kr[b2][1],
                          kr[b2][2], kr[b2][3]);
#pragma unroll
                for (int ks = 0; ks < kKSteps; ++ks) {
                  const uint32_t r_lo = kr[ks >> 1][(ks & 1) * 2], r_hi = kr[ks >> 1][(ks & 1) * 2 + 1];
                  uint32_t kf[4];
                  kf[0] = e4m3x2_to_f16x2(r_lo);         // token r8,   d 4qc, 4qc+1
                  kf[1] = e4m3x2_to_f16x2(r_hi);         // token r8+8
                  kf[2] = e4m3x2_to_f16x2(r_lo >> 16);   // token r8,   d 4qc+2, 4qc+3
                  kf[3] = e4m3x2_to_f16x2(r_hi >> 16);   // token r8+8
#pragma unroll
                  for (int ht = 0; ht < kHT; ++ht)
                    mma_f16_16816(sacc[pg][ht], kf, qb[ht][ks][0], qb[ht][ks][1]);
                }
              } else {
                uint32_t kf[kKSteps][4];
#pragma unroll
                for (int ks = 0; ks < kKSteps; ++ks) {
                  const int col = ks * 16 + (mi >> 1) * 8;
                  ldsm_x4(sw128_addr(kbase + (col >> 6) * L::kBoxBytes, tok, col & 63), kf[ks][0],
                          kf[ks][1], kf[ks][2], kf[ks][3]);
                }
#pragma unroll
                for (int ks = 0; ks < kKSteps; ++ks)
#pragma unroll
                  for (int ht = 0; ht < kHT; ++ht)
                    mma_bf16_16816(sacc[pg][ht], kf[ks], qb[ht][ks][0], qb[ht][ks][1]);
              }
            }
          }
        }
        // ---- online softmax per head over this step's tokens; tokens past
        // the sequence end -> -inf.  sc[pg][ht][i]: i = e (token r8, head 2qc+e)
        // and 2+e (token r8+8)
        uint32_t pbf[2][kHT][2];   // P^T fragments (B operand) per page and head tile
        float alpha[kHT][2];
#pragma unroll
        for (int ht = 0; ht < kHT; ++ht) {
          float sc[2][4];
#pragma unroll
          for (int pg = 0; pg < kPPW; ++pg)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int tok = r8 + (i >> 1) * 8;
              sc[pg][i] = tok < valid[pg] ? sacc[pg][ht][i] * sl2 : -INFINITY;
            }
          float e[2][4];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float mx = fmaxf(sc[0][hh], sc[0][2 + hh]);
            if (kPPW == 2) mx = fmaxf(mx, fmaxf(sc[1][hh], sc[1][2 + hh]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run[ht][hh], mx);
            alpha[ht][hh] = fast_exp2(m_run[ht][hh] - m_new);   // 0 on the first step
            m_run[ht][hh] = m_new;
#pragma unroll
            for (int pg = 0; pg < kPPW; ++pg) {
              e[pg][hh] = fast_exp2(sc[pg][hh] - m_new);
              e[pg][2 + hh] = fast_exp2(sc[pg][2 + hh] - m_new);
            }
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            l_run[ht][hh] *= alpha[ht][hh];
            le_run[ht][hh] *= alpha[ht][hh];
          }
#pragma unroll
          for (int pg = 0; pg < kPPW; ++pg) {
            // rows r8 (lo) and r8+8 (hi) of S^T as 16-bit pairs (heads 2qc,
            // 2qc+1): bf16, or f16 for the FP8 cache.  O is normalised by the
            // rounded weights that feed P.V; the LSE uses the exact ones
            // (the rounded halves are added by the mixed-precision add)
            uint32_t lo, hi;
            if constexpr (kFp8) {
              lo = pack_f16x2(e[pg][0], e[pg][1]);
              hi = pack_f16x2(e[pg][2], e[pg][3]);
              add_f16x2_to_f32(l_run[ht][0], l_run[ht][1], lo);
              add_f16x2_to_f32(l_run[ht][0], l_run[ht][1], hi);
            } else {
              lo = pack_bf16x2(e[pg][0], e[pg][1]);
              hi = pack_bf16x2(e[pg][2], e[pg][3]);
              add_bf16x2_to_f32(l_run[ht][0], l_run[ht][1], lo);
              add_bf16x2_to_f32(l_run[ht][0], l_run[ht][1], hi);
            }
            le_run[ht][0] += e[pg][0] + e[pg][2];
            le_run[ht][1] += e[pg][1] + e[pg][3];
            // transpose to the B layout of P^T (token pairs, head r8)
            pbf[pg][ht][0] = movmatrix_trans(lo);
            pbf[pg][ht][1] = movmatrix_trans(hi);
          }
        }
        bool any_scale = false;
#pragma unroll
        for (int ht = 0; ht < kHT; ++ht) any_scale |= (alpha[ht][0] != 1.f) || (alpha[ht][1] != 1.f);
        if (__any_sync(0xffffffffu, any_scale)) {
#pragma unroll
          for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
            for (int ht = 0; ht < kHT; ++ht) {
              acc[mt][ht][0] *= alpha[ht][0];
              acc[mt][ht][1] *= alpha[ht][1];
              acc[mt][ht][2] *= alpha[ht][0];
              acc[mt][ht][3] *= alpha[ht][1];
            }
        }
        // ---- O^T += V^T.P^T per page: V^T fragments by transposing ldmatrix
        if constexpr (kFp8) {
          // matrix mi: tokens (mi&1)*8.., 16-byte chunk 2u + (mi>>1).  A
          // transposed word holds tokens 2qc, 2qc+1 of d pair (2r8, 2r8+1);
          // the byte permute splits it into the even-d pair (row r8 of the
          // m-tile) and the odd-d pair (row r8+8)
          const int mi = lane >> 3, j = lane & 7;
          const int tok = (mi & 1) * 8 + j;
#pragma unroll
          for (int pg = 0; pg < kPPW; ++pg) {
            if (pg < npg) {
              const uint32_t vbase = base + pg * 2 * L::kPageBytes + L::kPageBytes;
              uint32_t vr[kMT / 2][4];
#pragma unroll
              for (int u = 0; u < kMT / 2; ++u)
                ldsm_x4_trans(sw128_chunk(vbase, tok, 2 * u + (mi >> 1)), vr[u][0], vr[u][1],
                              vr[u][2], vr[u][3]);
              const int v = valid[pg];
              const int t0 = 2 * qc;
              const uint32_t m01 = (t0 < v ? 0xffffu : 0u) | (t0 + 1 < v ? 0xffff0000u : 0u);
              const uint32_t m89 = (t0 + 8 < v ? 0xffffu : 0u) | (t0 + 9 < v ? 0xffff0000u : 0u);
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt) {
                const uint32_t w0 = prmt_b32(vr[mt >> 1][(mt & 1) * 2], 0x3120u);       // tokens 2qc..
                const uint32_t w8 = prmt_b32(vr[mt >> 1][(mt & 1) * 2 + 1], 0x3120u);   // tokens 8+2qc..
                uint32_t vf[4];
                vf[0] = e4m3x2_to_f16x2(w0);          // d 16mt + 2r8,     tokens 2qc, 2qc+1
                vf[1] = e4m3x2_to_f16x2(w0 >> 16);    // d 16mt + 2r8 + 1
                vf[2] = e4m3x2_to_f16x2(w8);          // d 16mt + 2r8,     tokens 8+2qc, 9+2qc
                vf[3] = e4m3x2_to_f16x2(w8 >> 16);    // d 16mt + 2r8 + 1
                if (v < kDecPage) {   // tokens past the sequence end may hold anything (NaN)
                  vf[0] &= m01;
                  vf[1] &= m01;
                  vf[2] &= m89;
                  vf[3] &= m89;
                }
#pragma unroll
                for (int ht = 0; ht < kHT; ++ht)
                  mma_f16_16816(acc[mt][ht], vf, pbf[pg][ht][0], pbf[pg][ht][1]);
              }
            }
          }
        } else         {
          const int mi = lane >> 3, j = lane & 7;
          const int tok = (mi >> 1) * 8 + j;
#pragma unroll
          for (int pg = 0; pg < kPPW; ++pg) {
            if (pg < npg) {
              const uint32_t vbase = base + pg * 2 * L::kPageBytes + L::kPageBytes;
              uint32_t vf[kMT][4];
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt) {
                const int col = mt * 16 + (mi & 1) * 8;
                ldsm_x4_trans(sw128_addr(vbase + (col >> 6) * L::kBoxBytes, tok, col & 63),
                              vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3]);
              }
              const int v = valid[pg];
              if (v < kDecPage) {   // tokens past the sequence end may hold anything (NaN)
                const int t0 = 2 * qc;
                const uint32_t m01 = (t0 < v ? 0xffffu : 0u) | (t0 + 1 < v ? 0xffff0000u : 0u);
                const uint32_t m89 = (t0 + 8 < v ? 0xffffu : 0u) | (t0 + 9 < v ? 0xffff0000u : 0u);
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                  vf[mt][0] &= m01;
                  vf[mt][1] &= m01;
                  vf[mt][2] &= m89;
                  vf[mt][3] &= m89;
                }
              }
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                for (int ht = 0; ht < kHT; ++ht)
                  mma_bf16_16816(acc[mt][ht], vf[mt], pbf[pg][ht][0], pbf[pg][ht][1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[stage]);
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }

    // ---- combine the warps' states in registers, halving the number of
    // holders each level (warps [n/2, n) send to [0, n/2))
    // stop together if any warp gave up (every consumer gets the same answer)
    if (bar_sync_or(1, kDecWarps * 32, !ok || abort_flag)) break;
    constexpr int kAccF = kMT * kHT * 4;
#pragma unroll
    for (int senders = kDecWarps / 2; senders >= 1; senders >>= 1) {
      if (cw >= senders && cw < 2 * senders) {
        float* dst = scratch + (cw - senders) * L::kFragFloats * 32 + lane;
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
          for (int ht = 0; ht < kHT; ++ht)
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[((mt * kHT + ht) * 4 + i) * 32] = acc[mt][ht][i];
#pragma unroll
        for (int ht = 0; ht < kHT; ++ht)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            dst[(kAccF + ht * 6 + hh) * 32] = m_run[ht][hh];
            dst[(kAccF + ht * 6 + 2 + hh) * 32] = l_run[ht][hh];
            dst[(kAccF + ht * 6 + 4 + hh) * 32] = le_run[ht][hh];
          }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32));
      if (cw < senders) {
        const float* src = scratch + cw * L::kFragFloats * 32 + lane;
        float wa[kHT][2], wb[kHT][2];
#pragma unroll
        for (int ht = 0; ht < kHT; ++ht)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float mo = src[(kAccF + ht * 6 + hh) * 32];
            const float mn = fmaxf(m_run[ht][hh], mo);
            // a state that saw no key has m = -inf and contributes nothing
            wa[ht][hh] = (m_run[ht][hh] == -INFINITY) ? 0.f : fast_exp2(m_run[ht][hh] - mn);
            wb[ht][hh] = (mo == -INFINITY) ? 0.f : fast_exp2(mo - mn);
            m_run[ht][hh] = mn;
            l_run[ht][hh] = l_run[ht][hh] * wa[ht][hh] + src[(kAccF + ht * 6 + 2 + hh) * 32] * wb[ht][hh];
            le_run[ht][hh] = le_run[ht][hh] * wa[ht][hh] + src[(kAccF + ht * 6 + 4 + hh) * 32] * wb[ht][hh];
          }
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
          for (int ht = 0; ht < kHT; ++ht)
#pragma unroll
            for (int i = 0; i < 4; ++i)
              acc[mt][ht][i] = acc[mt][ht][i] * wa[ht][i & 1] +
                               src[((mt * kHT + ht) * 4 + i) * 32] * wb[ht][i & 1];
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32));
    }

    // ---- warp 0 writes the piece: the final rows, or one partial (cluster
    // mode: this CTA's state, into its own shared memory)
    const int seg = pc.b * nseg_b + pc.seg_in_b;
    const bool whole = kCluster ? (cl_size == 1) : (pc.pg0 == 0) && (pc.pg1 == pc.npg);
    const int slot = c + seg;
    if (kCluster && !whole) {
      if (cw == 0) {
#pragma unroll
        for (int ht = 0; ht < kHT; ++ht)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float ls = l_run[ht][hh], le = le_run[ht][hh];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
              ls += __shfl_xor_sync(0xffffffffu, ls, off);
              le += __shfl_xor_sync(0xffffffffu, le, off);
            }
            const int r = ht * 8 + 2 * qc + hh;   // head within the segment
            float* xo = scratch + L::kXchO + r * D;
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
              xo[mt * 16 + r8] = acc[mt][ht][hh];
              xo[mt * 16 + 8 + r8] = acc[mt][ht][2 + hh];
            }
            if (r8 == 0)
              *reinterpret_cast<float4*>(scratch + L::kXchS + 4 * r) =
                  make_float4(m_run[ht][hh], ls, le, 0.f);
          }
      }
    } else if (cw == 0) {
#pragma unroll
      for (int ht = 0; ht < kHT; ++ht)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // each head's sums are spread over the 8 lanes with the same qc
          float ls = l_run[ht][hh], le = le_run[ht][hh];
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            ls += __shfl_xor_sync(0xffffffffu, ls, off);
            le += __shfl_xor_sync(0xffffffffu, le, off);
          }
          const int r = ht * 8 + 2 * qc + hh;   // head within the segment
          if (r < nh) {
            const float inv = o_scale / ls;
            const float lse2 = m_run[ht][hh] + fast_log2(le);
            // m-tile row r8 / r8+8 is d 16mt + r8 / + 8 (bf16 cache), or the
            // pair d 16mt + 2r8, + 1 (FP8 cache)
            if (whole) {
              __nv_bfloat16* orow = p.o + ((size_t)pc.b * p.Hq + h0 + r) * D;
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt) {
                if constexpr (kFp8) {
                  *reinterpret_cast<uint32_t*>(orow + mt * 16 + 2 * r8) =
                      pack_bf16x2(acc[mt][ht][hh] * inv, acc[mt][ht][2 + hh] * inv);
                } else {
                  orow[mt * 16 + r8] = __float2bfloat16(acc[mt][ht][hh] * inv);
                  orow[mt * 16 + 8 + r8] = __float2bfloat16(acc[mt][ht][2 + hh] * inv);
                }
              }
              if (r8 == 0 && p.lse != nullptr) p.lse[(size_t)pc.b * p.Hq + h0 + r] = lse2 * kLn2;
            } else {
              float* orow = p.ws_o + ((size_t)slot * kDecHeadsPerSeg + r) * D;
#pragma unroll
              for (int mt = 0; mt < kMT; ++mt) {
                if constexpr (kFp8) {
                  *reinterpret_cast<float2*>(orow + mt * 16 + 2 * r8) =
                      make_float2(acc[mt][ht][hh] * inv, acc[mt][ht][2 + hh] * inv);
                } else {
                  orow[mt * 16 + r8] = acc[mt][ht][hh] * inv;
                  orow[mt * 16 + 8 + r8] = acc[mt][ht][2 + hh] * inv;
                }
              }
              if (r8 == 0) p.ws_lse[(size_t)slot * kDecHeadsPerSeg + r] = lse2;
            }
          }
        }
      // the owner of the segment's first page records where its pieces are
      // (cluster mode has no workspace: a one-CTA cluster writes its rows whole)
      if (!kCluster && pc.pg0 == 0 && lane == 0)
        p.ws_seg[seg] = whole ? make_int2(-1, -1) : make_int2(c, dec_cta_of(pc.seg_u0 + pc.npg - 1, T, C));
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32));   // scratch reuse
  } while (next_piece(pc));
  }   // consumers

  if constexpr (kCluster) {
    if (cl_size > 1) {
      // ---- merge of the cluster's states (log-sum-exp, as in the
      // cross-warp combine): o = sum_c 2^(m_c - M) acc_c / sum_c 2^(m_c - M) l_c,
      // lse = M + log2 sum_c 2^(m_c - M) le_c.  Each thread of the cluster
      // takes float4 columns of the segment's rows.
      cluster_sync();   // every CTA's state is in its shared memory
      {
        const int seg_in_b = cl_seg % nseg_b;
        const int b = cl_seg / nseg_b;
        const int kvh = seg_in_b / p.hgroups;
        const int h0 = kvh * p.g + (seg_in_b % p.hgroups) * kDecHeadsPerSeg;
        const int nh = min(kDecHeadsPerSeg, p.g - (seg_in_b % p.hgroups) * kDecHeadsPerSeg);
        constexpr int kV4 = D / 4;
        constexpr float kLn2 = 0.69314718055994530942f;
        // item = (head r, float4 column l4), dealt round-robin over the
        // cluster's CTAs first, so every CTA merges an equal part; each thread
        // issues all of its remote loads (every CTA's abort flag and state)
        // before using any of them, so an item costs one round trip
        for (int it = cl_rank + cl_size * (int)threadIdx.x; it < nh * kV4;
             it += cl_size * (int)blockDim.x) {
          const int r = it / kV4, l4 = it % kV4;
          float4 sc[16], oc[16];   // {m, l, l_exact, -} and the o columns of each CTA
          int gave_up = 0;
#pragma unroll
          for (int q2 = 0; q2 < 16; ++q2) {
            if (q2 < cl_size) {
              gave_up |= dsmem_ld_s32(dsmem_addr(&abort_flag, (uint32_t)q2));
              sc[q2] = dsmem_ld_f32x4(dsmem_addr(scratch + L::kXchS + 4 * r, (uint32_t)q2));
              oc[q2] = dsmem_ld_f32x4(dsmem_addr(scratch + L::kXchO + r * D + 4 * l4, (uint32_t)q2));
            }
          }
          if (gave_up) break;   // a CTA of the cluster stopped on a device error
          float M = -INFINITY;
#pragma unroll
          for (int q2 = 0; q2 < 16; ++q2)
            if (q2 < cl_size) M = fmaxf(M, sc[q2].x);
          float ls = 0.f, le = 0.f;
          float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int q2 = 0; q2 < 16; ++q2) {
            if (q2 < cl_size) {
              // a CTA that saw no key (m = -inf) adds nothing
              const float w = (sc[q2].x == -INFINITY) ? 0.f : fast_exp2(sc[q2].x - M);
              ls += w * sc[q2].y;
              le += w * sc[q2].z;
              o4.x += w * oc[q2].x;
              o4.y += w * oc[q2].y;
              o4.z += w * oc[q2].z;
              o4.w += w * oc[q2].w;
            }
          }
          const float inv = ls > 0.f ? 1.f / ls : 0.f;
          const size_t row = (size_t)b * p.Hq + h0 + r;
          *reinterpret_cast<uint2*>(p.o + row * D + 4 * l4) =
              make_uint2(pack_bf16x2(o4.x * inv, o4.y * inv), pack_bf16x2(o4.z * inv, o4.w * inv));
          if (l4 == 0 && p.lse != nullptr) p.lse[row] = (M + fast_log2(le)) * kLn2;
        }
      }
      cluster_sync();   // no CTA leaves while another still reads its shared memory
    }
  }
}

// Log-sum-exp merge of split segments' partials: o = sum_c 2^(lse_c - M) o_c /
// sum_c 2^(lse_c - M), lse = M + log2 of that denominator, over the CTAs c that
// held a piece of the segment (M = max lse_c).  Rows are (sequence, query
// head); CTA x takes rows x, x + grid, ... and first finds, in parallel,
// which of them belong to split segments and how many parts the largest has.
// A thread group (one float4 of a row per thread) reduces its parts in one
// pass with a running maximum.  Each row gets gpr groups -- enough that a
// group has at most four parts, so its loads go out together -- and the CTA
// works on kGroups / gpr rows at once; a row's groups are then combined
// through shared memory.
constexpr int kMergeThreads = 512;

template <int D>
__global__ void __launch_bounds__(kMergeThreads, 2) decode_merge_kernel(const DecodeParams p) {
  constexpr int kV = D / 4;                    // float4 per row
  constexpr int kGroups = kMergeThreads / kV;  // thread groups (16 at D = 128)
  constexpr float kLn2 = 0.69314718055994530942f;
  __shared__ float4 red[kGroups][kV];
  __shared__ float red_m[kGroups], red_s[kGroups];
  __shared__ int list[kMergeThreads];
  __shared__ int2 range[kMergeThreads];         // CTAs holding the row's pieces
  __shared__ int prefix[kDecMaxBatch + 1];      // page prefix over the batch
  __shared__ int nlist, max_parts;

  const int t = threadIdx.x, grp = t / kV, l = t % kV;
  const int nseg_b = p.Hkv * p.hgroups;
  const long long rows = (long long)p.B * p.Hq;
  auto seg_of = [&](int row, int& r) {
    const int b = row / p.Hq, h = row % p.Hq;
    const int kvh = h / p.g, hq = h % p.g;
    r = hq % kDecHeadsPerSeg;
    return b * nseg_b + kvh * p.hgroups + hq / kDecHeadsPerSeg;
  };
  // Which rows were split, and over which CTAs, follows from the sequence
  // lengths and the streaming kernel's plan alone (the same page prefix and
  // equal shares of the unit line), so it is worked out before waiting for
  // that kernel: the lengths are an input of the call, which the streaming
  // kernel never writes, and were final before it started.
  if (t < 32) {
    const int per = (p.B + 31) / 32, b0 = t * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (b0 + i < p.B) local += dec_pages_of(p, b0 + i);
    int incl = local;
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (t >= off) incl += v;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i)
      if (b0 + i < p.B) {
        prefix[b0 + i] = run;
        run += dec_pages_of(p, b0 + i);
      }
    if (t == 31) prefix[p.B] = incl;
  }
  __syncthreads();
  const long long T = (long long)prefix[p.B] * nseg_b;   // the streaming kernel's unit line
  const int C = (int)min((long long)p.parts, T);          // its CTAs with a non-empty share
  auto build_list = [&](long long base) {
    if (t == 0) {
      nlist = 0;
      max_parts = 1;
    }
    __syncthreads();
    const long long row = blockIdx.x + (base + t) * gridDim.x;
    if (row < rows) {
      const int b = (int)(row / p.Hq);
      const int npg = prefix[b + 1] - prefix[b];
      if (npg > 0) {   // (an empty sequence's rows were written by the streaming kernel)
        int r;
        const int seg_in_b = seg_of((int)row, r) - b * nseg_b;
        const long long seg_u0 = (long long)prefix[b] * nseg_b + (long long)seg_in_b * npg;
        const int first = dec_cta_of(seg_u0, T, C), last = dec_cta_of(seg_u0 + npg - 1, T, C);
        if (first != last) {   // split: pieces in CTAs first..last
          const int k = atomicAdd(&nlist, 1);
          list[k] = (int)row;
          range[k] = make_int2(first, last);
          atomicMax(&max_parts, last - first + 1);
        }
      }
    }
    __syncthreads();
  };
  build_list(0);
  griddep_wait();   // the streaming kernel's partials
  griddep_launch_dependents();

  for (long long base = 0; blockIdx.x + base * gridDim.x < rows; base += kMergeThreads) {
    if (base > 0) build_list(base);
    const int n = nlist;
    int gpr = 1;   // groups per row: a power of two with gpr * 4 >= parts
    while (gpr < kGroups && gpr * 4 < max_parts) gpr <<= 1;
    const int rpp = kGroups / gpr;               // rows per pass
    const int slot = grp / gpr, sub = grp % gpr;
    for (int k0 = 0; k0 < n; k0 += rpp) {
      const int k = k0 + slot;
      float m = -INFINITY, S = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int row_k = -1, seg = 0, r = 0;
      if (k < n) {
        row_k = list[k];
        seg = seg_of(row_k, r);
        const int2 info = range[k];
        // parts sub, sub + gpr, ... in batches of four whose loads are all
        // issued before any is used; every part holds at least one key, so
        // its LSE is finite (-inf marks a slot past the last part)
        for (int c0 = info.x + sub; c0 <= info.y; c0 += 4 * gpr) {
          float x[4];
          float4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int cc = c0 + j * gpr;
            x[j] = -INFINITY;
            v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (cc <= info.y) {
              const size_t sl = (size_t)(cc + seg) * kDecHeadsPerSeg + r;
              x[j] = p.ws_lse[sl];
              v[j] = reinterpret_cast<const float4*>(p.ws_o + sl * D)[l];
            }
          }
          const float mn = fmaxf(fmaxf(m, fmaxf(x[0], x[1])), fmaxf(x[2], x[3]));
          const float a = fast_exp2(m - mn);   // 0 while m = -inf
          S *= a;
          acc.x *= a;
          acc.y *= a;
          acc.z *= a;
          acc.w *= a;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float w = fast_exp2(x[j] - mn);   // 0 for an empty slot
            S += w;
            acc.x += w * v[j].x;
            acc.y += w * v[j].y;
            acc.z += w * v[j].z;
            acc.w += w * v[j].w;
          }
          m = mn;
        }
      }
      red[grp][l] = acc;
      if (l == 0) {
        red_m[grp] = m;
        red_s[grp] = S;
      }
      __syncthreads();
      if (sub == 0 && row_k >= 0) {
        // the row's first group combines the row's gpr groups
        float M = -INFINITY;
        for (int g2 = grp; g2 < grp + gpr; ++g2) M = fmaxf(M, red_m[g2]);
        float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
        float St = 0.f;
        for (int g2 = grp; g2 < grp + gpr; ++g2) {
          const float mg = red_m[g2];
          const float w = mg == -INFINITY ? 0.f : fast_exp2(mg - M);   // a group with no part
          const float4 v = red[g2][l];
          o4.x += w * v.x;
          o4.y += w * v.y;
          o4.z += w * v.z;
          o4.w += w * v.w;
          St += w * red_s[g2];
        }
        const float inv = 1.f / St;
        *reinterpret_cast<uint2*>(p.o + (size_t)row_k * D + 4 * l) =
            make_uint2(pack_bf16x2(o4.x * inv, o4.y * inv), pack_bf16x2(o4.z * inv, o4.w * inv));
        if (l == 0 && p.lse != nullptr) p.lse[row_k] = (M + fast_log2(St)) * kLn2;
      }
      __syncthreads();   // red, red_m, red_s reuse
    }
  }
}

}  // namespace frt
