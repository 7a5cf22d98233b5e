// Split-K MLA decode attention over the paged latent cache (weight-absorbed form).
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": per token and layer the cache keeps the 512-dim latent c_kv
//      and the 64-dim rope key; kv_b_proj (512 -> 32 x (128 + 128)) expands K_nope
//      and V per head at attention time.  The absorbed form moves W_UK onto the
//      query and W_UV after the probability-weighted latent sum, so the cache is
//      read once as [c_kv | k_pe] rows.
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 二: the KV
//      cache, not the weights, is what long contexts pay for; reading it is the
//      whole cost of a decode step.
//
// One CTA per (sequence, row group, KV split): 64-token pages are streamed by
// TMA into a shared-memory ring; S^T = page . q_ext^T (M = 64 tokens, N = rows,
// K = 576) and O^T += c_kv^T . P^T (M = 128 latent dims x 4, N = rows, K = 64
// tokens) run on tcgen05 with fp32 accumulators in tensor memory; S is
// double-buffered so the QK of page i+1 runs while the softmax of page i does;
// the online softmax (base 2, lazy max update) runs in registers.  Writes the
// split's (m, l, O); the combine kernel merges the splits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>

#include "split_kv.h"
#include "xmla_device.cuh"

namespace xmla {

// A row's running maximum is only raised when a score exceeds it by more than
// this (log2 units), so probabilities stay <= 2^kLazyMax before normalisation.
constexpr float kLazyMax = 8.0f;
constexpr int kSoftmaxThreads = 128;
constexpr int kSoftmaxWarp0 = 3;  // warps: 0 TMA producer, 1 QK issuer, 2 PV issuer, 3-6 softmax
constexpr int kDecodeThreads = 32 * kSoftmaxWarp0 + kSoftmaxThreads;

// ---------------------------------------------------------------- shared-memory plan

// kSplitQ (32 rows only): q_ext comes as two bf16 rows per query row, hi and
// lo = bf16(q - hi), so the QK product carries ~16 bits of the query: the
// product runs with N = 64 (rows hi 0..31, lo 32..63) and the softmax adds
// the two halves of S.  Otherwise q_ext is a single bf16 row each.  The split
// needs 36 KB more of shared memory, taken from the page ring.
// P^T buffers with 64 rows per CTA (two where shared memory allows)
constexpr int kPBufs64 = 2;

template <int NR, bool kSplitQ_ = false>
struct DecodeLayout {
  static_assert(NR == 32 || NR == 64, "rows per CTA");
  static_assert(NR == 32 || !kSplitQ_, "the split query needs 32 rows per CTA");
  static constexpr bool kSplitQ = kSplitQ_;
  static constexpr int kQRows = kSplitQ ? 2 * NR : NR;  // B rows of the QK product
  // 16 KB latent slots (dims 128m..128m+127 of a page) and 8 KB rope slots.
  // At least two pages of latent slots, so page i + 1 never waits for a slot
  // of page i (whose PV needs page i's softmax); with 64 rows that leaves room
  // for one rope slot, which the QK product then reads first and frees early.
  static constexpr int kLatSlots = NR == 32 && !kSplitQ ? 9 : 8;
  static constexpr int kRopeSlots = NR == 32 ? (kSplitQ ? 2 : 4) : 1;
  static constexpr bool kRopeFirst = kRopeSlots == 1;
  static constexpr uint32_t kQChunk = kQRows * 128;    // one 64-column chunk of q_ext
  // P^T is stored MN-major: one row of NR bf16 per token, 64 B (64-byte swizzle)
  // for 32 rows or 128 B (128-byte swizzle) for 64 rows.
  static constexpr uint32_t kPRow = NR * 2;
  static constexpr uint32_t kPBytes = 64 * kPRow;
  static constexpr uint32_t kPSwizzle = NR == 32 ? kSwizzle64B : kSwizzle128B;
  static constexpr uint32_t kPGroup = 8 * kPRow;       // 8 tokens: one swizzle atom
  static constexpr uint32_t kLatBytes = 16384;
  static constexpr uint32_t kRopeBytes = 8192;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffP = kOffQ + 9 * kQChunk;
  static constexpr int kPBufs = NR == 32 ? 2 : kPBufs64;
  static constexpr uint32_t kOffLat = kOffP + kPBufs * kPBytes;
  static constexpr uint32_t kOffRope = kOffLat + kLatSlots * kLatBytes;
  static constexpr uint32_t kOffBars = kOffRope + kRopeSlots * kRopeBytes;
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarLatFull = 1;
  static constexpr int kBarLatEmpty = kBarLatFull + kLatSlots;
  static constexpr int kBarRopeFull = kBarLatEmpty + kLatSlots;
  static constexpr int kBarRopeEmpty = kBarRopeFull + kRopeSlots;
  static constexpr int kBarSFull = kBarRopeEmpty + kRopeSlots;  // 2
  static constexpr int kBarSFree = kBarSFull + 2;               // 2
  static constexpr int kBarPFull = kBarSFree + 2;               // 2
  static constexpr int kBarPvDone = kBarPFull + 2;              // 2
  static constexpr int kBarDrain = kBarPvDone + 2;  // 2: QK issuer, PV issuer
  static constexpr int kNumBars = kBarDrain + 2;
  static constexpr uint32_t kOffMUsed = (kOffBars + kNumBars * 8 + 15) & ~15u;
  static constexpr uint32_t kOffMNext = kOffMUsed + NR * 4;
  static constexpr uint32_t kOffAlpha = kOffMNext + NR * 4;
  static constexpr uint32_t kOffRed = kOffAlpha + NR * 4;
  static constexpr uint32_t kOffTmem = kOffRed + 4 * NR * 4;
  static constexpr uint32_t kOffAbort = kOffTmem + 4;
  static constexpr uint32_t kBytes = kOffAbort + 12;
  static constexpr uint32_t kSmem = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(kOffP % 1024 == 0 && kOffLat % 1024 == 0 && kOffRope % 1024 == 0, "alignment");
  // tensor memory columns: O^T at [0, 4 NR), S^T buffers of kSCols columns after it
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = 4 * NR;
  static constexpr uint32_t kSCols = kQRows;  // columns of one S^T buffer
  static constexpr uint32_t kTmemCols = 4 * NR + 2 * kSCols <= 256 ? 256 : 512;
};


// Warp transpose-reduction: on return v[0] of lane L holds the reduction over
// the 32 lanes of input row L (31 shuffles for 32 rows).
template <bool kMax>
__device__ __forceinline__ void xpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int k = 0; k < w; ++k) {
      const float send = upper ? v[k] : v[k + w];
      const float keep = upper ? v[k + w] : v[k];
      const float recv = __shfl_xor_sync(0xffffffffu, send, w);
      v[k] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
}

// The same over the 16 threads of one row parity (lane bits 0, 2, 3, 4; bit 1
// kept): on return v[0] holds the reduction of value j = b0 + 2 b2 + 4 b3 + 8 b4.
template <bool kMax>
__device__ __forceinline__ void xpose_reduce16(float (&v)[16], int lane) {
  constexpr int kMask[4] = {16, 8, 4, 1};
#pragma unroll
  for (int lv = 0; lv < 4; ++lv) {
    const int w = 8 >> lv;  // values kept after this level
    const bool upper = (lane & kMask[lv]) != 0;
#pragma unroll
    for (int k = 0; k < w; ++k) {
      const float send = upper ? v[k] : v[k + w];
      const float keep = upper ? v[k + w] : v[k];
      const float recv = __shfl_xor_sync(0xffffffffu, send, kMask[lv]);
      v[k] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// How a CTA finds its pages.
enum WorkMode : int {
  kWorkSplit = 0,   // split (blockIdx % nsplit) of every sequence's pages
  kWorkRanged = 1,  // the same over the logical pages [p.page_lo, p.page_hi) of every sequence
                    // (one rank's share of a sequence-parallel decode)
  kWorkTable = 2,   // entry blockIdx of p.work_tab (written by the preceding kernel)
};

// What one pass of the split-K attention covers: queries [j0, j0 + jn) of
// sequence b (32 rows each) over its logical pages [p_begin, p_begin +
// n_pages); the split's partials go to rows [row0, row0 + 32 jn).
struct DecodePass {
  int b;
  int j0;
  int jn;
  int n_pages;
  int64_t seqlen;
  int64_t npages;   // pages of the whole sequence
  int64_t p_begin;
  int64_t row0;     // first partial row
  int32_t qrow0;    // first q_ext row loaded for the QK product
};

// Barrier initialisation of one pass (one thread); clears the abort flag.
// `bars`: shared address of the pass's barrier set (L::kNumBars words).
template <int NR, bool kSplitQ>
__device__ __forceinline__ void decode_init_barriers(uint32_t bars, volatile int* abort_flag) {
  using L = DecodeLayout<NR, kSplitQ>;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  mbar_init(bar(L::kBarQ), 1);
  for (int i = 0; i < L::kLatSlots; ++i) {
    mbar_init(bar(L::kBarLatFull + i), 1);
    mbar_init(bar(L::kBarLatEmpty + i), 1);
  }
  for (int i = 0; i < L::kRopeSlots; ++i) {
    mbar_init(bar(L::kBarRopeFull + i), 1);
    mbar_init(bar(L::kBarRopeEmpty + i), 1);
  }
  for (int i = 0; i < 2; ++i) {
    mbar_init(bar(L::kBarSFull + i), 1);
    mbar_init(bar(L::kBarSFree + i), kSoftmaxThreads);
    mbar_init(bar(L::kBarPFull + i), kSoftmaxThreads);
    mbar_init(bar(L::kBarPvDone + i), 1);
  }
  mbar_init(bar(L::kBarDrain + 0), 1);
  mbar_init(bar(L::kBarDrain + 1), 1);
  *abort_flag = 0;
  fence_barrier_init();
}

// The roles of a CTA over one pass (DecodePass): warp 0 streams the pages by
// TMA, warp 1 issues QK, warp 2 issues PV, warps 3-6 run the softmax and write
// the split's (m, l, O).  The caller initialises the barrier set at `bars`
// (decode_init_barriers) and allocates tensor memory.
// kQHiRows (single query only): q_ext is in the split layout and the pass
// uses the hi rows alone, query k of the pass at row qrow0 + 64 k (32-row
// boxes; a 32-row box lands with the same 128-byte swizzle phase as the
// corresponding half of a 64-row one, the halves being 4 KB apart).
template <int NR, bool kSplitQ, bool kQHiRows = false>
__device__ __forceinline__ void decode_pass(uint8_t* smem, uint32_t base, uint32_t bars,
                                            uint32_t tmem_base, const CUtensorMap& tmap_pool,
                                            const CUtensorMap& tmap_q, const DecodeParams& p,
                                            const DecodePass& w) {
  using L = DecodeLayout<NR, kSplitQ>;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
  float* m_used = reinterpret_cast<float*>(smem + L::kOffMUsed);
  float* m_next = reinterpret_cast<float*>(smem + L::kOffMNext);
  float* alpha_s = reinterpret_cast<float*>(smem + L::kOffAlpha);
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = w.b;
  const int64_t seqlen = w.seqlen, npages = w.npages, p_begin = w.p_begin;
  const int j0 = w.j0, jn = w.jn, nrows = jn * 32, n_pages = w.n_pages;
  const int32_t qrow0 = w.qrow0;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0 && n_pages > 0) {
      tma_prefetch_desc(&tmap_pool);
      tma_prefetch_desc(&tmap_q);
      // Pages are read once at q_len 1: evict them first.  With two row groups
      // (q_len > 1) both groups' CTAs stream the same pages at about the same
      // time, and the second read should find them in L2.
      const uint64_t stream_policy = NR == 32 ? policy_evict_first() : policy_evict_normal();
      int li = 0, ri = 0;
      uint32_t lph = 0, rph = 0;
      int64_t lat_issued = 0, rope_issued = 0;
      bool ok = true;
      // block ids are fetched four pages ahead so their load latency is hidden
      const int32_t* bt = p.block_table + (int64_t)b * p.max_blocks + p_begin;
      int32_t nb0 = bt[0];
      int32_t nb1 = n_pages > 1 ? bt[1] : 0;
      int32_t nb2 = n_pages > 2 ? bt[2] : 0;
      int32_t nb3 = n_pages > 3 ? bt[3] : 0;
      // q_ext, the rows this step appends, and any cache rows an earlier kernel
      // on the stream may still be writing: all of them are read only after
      // the kernels launched before have completed.  (This CTA could only start
      // once the previous kernel's CTAs had left its SM, so the wait is short.)
      // q_ext is loaded first, so the first QK product waits only for its page.
      pdl_wait();
      mbar_arrive_expect_tx(bar(L::kBarQ), 9u * L::kQChunk);
      for (int c = 0; c < 9; ++c)
        if constexpr (kQHiRows) {
#pragma unroll
          for (int k = 0; k < NR / 32; ++k)
            tma_load_2d(base + L::kOffQ + c * L::kQChunk + k * 4096u, &tmap_q, c * 64,
                        qrow0 + 64 * k, bar(L::kBarQ));
        } else {
          tma_load_2d(base + L::kOffQ + c * L::kQChunk, &tmap_q, c * 64, qrow0, bar(L::kBarQ));
        }
      for (int i = 0; i < n_pages && ok; ++i) {
        int32_t blk = nb0;
        nb0 = nb1;
        nb1 = nb2;
        nb2 = nb3;
        nb3 = i + 4 < n_pages ? bt[i + 4] : 0;
        if (blk < 0 || (int64_t)blk >= p.num_blocks) {
          record_status(p.status, XMLA_ERR_DEVICE_OOB);
          blk = (int32_t)p.num_blocks;  // past the end: the tensor copy reads zeros
        }
        const int32_t y = blk * kPage;
        auto issue_rope = [&]() {
          if (!mbar_wait(bar(L::kBarRopeEmpty + ri), rph ^ 1u, abort_flag, p.status,
                         p.wait_limit_ns))
            return false;
          mbar_arrive_expect_tx(bar(L::kBarRopeFull + ri), L::kRopeBytes);
          tma_load_2d_hint(base + L::kOffRope + ri * L::kRopeBytes, &tmap_pool, kDLatent, y,
                           bar(L::kBarRopeFull + ri), stream_policy);
          ++rope_issued;
          if (++ri == L::kRopeSlots) { ri = 0; rph ^= 1u; }
          return true;
        };
        // the chunk the QK product reads first is requested first
        if constexpr (L::kRopeFirst) {
          if (!(ok = issue_rope())) break;
        }
        for (int m = 0; m < 4; ++m) {
          if (!mbar_wait(bar(L::kBarLatEmpty + li), lph ^ 1u, abort_flag, p.status,
                         p.wait_limit_ns)) {
            ok = false;
            break;
          }
          const uint32_t dst = base + L::kOffLat + li * L::kLatBytes;
          mbar_arrive_expect_tx(bar(L::kBarLatFull + li), L::kLatBytes);
          tma_load_2d_hint(dst, &tmap_pool, 128 * m, y, bar(L::kBarLatFull + li), stream_policy);
          tma_load_2d_hint(dst + 8192, &tmap_pool, 128 * m + 64, y, bar(L::kBarLatFull + li),
                           stream_policy);
          ++lat_issued;
          if (++li == L::kLatSlots) { li = 0; lph ^= 1u; }
        }
        if (!ok) break;
        if constexpr (!L::kRopeFirst) {
          if (!(ok = issue_rope())) break;
        }
      }
      // Every copy issued must land before the CTA may exit: wait for the last
      // phase armed on each slot (immediate when the consumer already saw it).
      mbar_wait(bar(L::kBarQ), 0, nullptr, p.status, p.wait_limit_ns);
      for (int s = 0; s < L::kLatSlots; ++s) {
        if (lat_issued > s) {
          const int64_t last = s + ((lat_issued - 1 - s) / L::kLatSlots) * L::kLatSlots;
          mbar_wait(bar(L::kBarLatFull + s), (uint32_t)((last / L::kLatSlots) & 1), nullptr,
                    p.status, p.wait_limit_ns);
        }
      }
      for (int s = 0; s < L::kRopeSlots; ++s) {
        if (rope_issued > s) {
          const int64_t last = s + ((rope_issued - 1 - s) / L::kRopeSlots) * L::kRopeSlots;
          mbar_wait(bar(L::kBarRopeFull + s), (uint32_t)((last / L::kRopeSlots) & 1), nullptr,
                    p.status, p.wait_limit_ns);
        }
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ================================================================ tensor-core issuers
    // Warp 1 issues QK (S^T[64 tok, NR] = page . q_ext^T into S buffer i & 1),
    // running up to two pages ahead of the softmax; warp 2 issues PV
    // (O^T[512, NR] += c_kv^T . P^T) as soon as a page's P is written.  Each
    // blocks in mbarrier try_wait, which suspends the thread instead of
    // spinning, so neither steals issue slots from the softmax warps.
    if (lane == 0 && n_pages > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(64, L::kQRows, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, NR, true, true);
      // descriptor bases; operands are reached by adding (byte offset >> 4)
      const uint64_t d_lat_k = smem_desc_sw128(base + L::kOffLat, 16, 1024);     // page, K-major
      const uint64_t d_rope_k = smem_desc_sw128(base + L::kOffRope, 16, 1024);
      const uint64_t d_q = smem_desc_sw128(base + L::kOffQ, 16, 1024);           // q_ext, K-major
      const uint64_t d_lat_mn = smem_desc_sw128(base + L::kOffLat, 8192, 1024);  // c_kv^T, MN-major
      const uint64_t d_p = smem_desc(base + L::kOffP, 8192, L::kPGroup, L::kPSwizzle);  // P^T, MN-major
      auto wait = [&](int idx, uint32_t parity) {
        return mbar_wait(bar(idx), parity, abort_flag, p.status, p.wait_limit_ns);
      };
      bool ok = true;
      if (warp == 1) {
        ok = wait(L::kBarQ, 0);
        tc_fence_after();
        for (int i = 0; i < n_pages && ok; ++i) {
          const int sb = i & 1;
          if (i >= 2) {
            if (!(ok = wait(L::kBarSFree + sb, (uint32_t)(((i - 2) >> 1) & 1)))) break;
            tc_fence_after();
          }
          const uint32_t t_s = tmem_base + L::kColS + sb * L::kSCols;
          const int r = i % L::kRopeSlots;
          if constexpr (L::kRopeFirst) {
            // the rope chunk first: its single slot is refilled for the next page
            // while this page's latent chunks go through
            if (!(ok = wait(L::kBarRopeFull + r, (uint32_t)((i / L::kRopeSlots) & 1)))) break;
            tc_fence_after();
            const uint64_t ar = d_rope_k + ((r * L::kRopeBytes) >> 4);
            const uint64_t bq = d_q + ((8 * L::kQChunk) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(t_s, ar + ((k * 32) >> 4), bq + ((k * 32) >> 4), idesc_qk, k != 0 ? 1u : 0u);
            tc_commit(bar(L::kBarRopeEmpty + r));
          }
          for (int m = 0; m < 4 && ok; ++m) {
            const int f = 4 * i + m;
            const int s = f % L::kLatSlots;
            if (!(ok = wait(L::kBarLatFull + s, (uint32_t)((f / L::kLatSlots) & 1)))) break;
            tc_fence_after();
            const uint64_t a0 = d_lat_k + ((s * L::kLatBytes) >> 4);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint64_t bq = d_q + (((2 * m + half) * L::kQChunk) >> 4);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                tc_mma_bf16(t_s, a0 + ((half * 8192 + k * 32) >> 4), bq + ((k * 32) >> 4), idesc_qk,
                            (L::kRopeFirst || (m | half | k) != 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          if constexpr (!L::kRopeFirst) {
            if (!(ok = wait(L::kBarRopeFull + r, (uint32_t)((i / L::kRopeSlots) & 1)))) break;
            tc_fence_after();
            const uint64_t ar = d_rope_k + ((r * L::kRopeBytes) >> 4);
            const uint64_t bq = d_q + ((8 * L::kQChunk) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(t_s, ar + ((k * 32) >> 4), bq + ((k * 32) >> 4), idesc_qk, 1u);
          }
          tc_commit(bar(L::kBarSFull + sb));
          if constexpr (!L::kRopeFirst) tc_commit(bar(L::kBarRopeEmpty + r));
        }
      } else {
        for (int i = 0; i < n_pages && ok; ++i) {
          if (!(ok = wait(L::kBarPFull + (i & 1), (uint32_t)((i >> 1) & 1)))) break;
          tc_fence_after();
          const uint64_t bp = d_p + (((i % L::kPBufs) * L::kPBytes) >> 4);
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
            const int s = (4 * i + m) % L::kLatSlots;
            const uint64_t a0 = d_lat_mn + ((s * L::kLatBytes) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(tmem_base + L::kColO + m * NR, a0 + ((k * 2048) >> 4),
                          bp + ((k * 2 * L::kPGroup) >> 4), idesc_pv, (i > 0 || k > 0) ? 1u : 0u);
            tc_commit(bar(L::kBarLatEmpty + s));
          }
          tc_commit(bar(L::kBarPvDone + (i & 1)));
        }
      }
      // all tensor-core work this thread issued must finish before tensor memory is freed
      const int drain = L::kBarDrain + (warp - 1);
      tc_commit(bar(drain));
      mbar_wait(bar(drain), 0, nullptr, p.status, p.wait_limit_ns);
    }
  } else {
    // ================================================================ softmax / epilogue
    // S^T of a page is an M=64 accumulator: page token r sits in tensor-memory
    // lane 32*(r/16) + r%16.  Each warp reads its quarter's 16 lanes with the
    // 16x64b shape, which spreads them over all 32 threads: thread t holds token
    // 8*(t&1) + (t>>2) of the quarter and the rows of one parity,
    // n = pr + 2j (pr = (t>>1)&1, j < NR/2).
    constexpr int kV = NR / 2;
    constexpr int kH = kV / 2;
    const int tid = threadIdx.x - 32 * kSoftmaxWarp0;
    const int quarter = warp & 3;            // tensor-memory lane quarter this warp may access
    const int pr = (lane >> 1) & 1;
    const int tok = 16 * quarter + 8 * (lane & 1) + (lane >> 2);  // token of the page
    // after a transposed butterfly over the 16 threads of one parity, value 0
    // of thread t belongs to row pr + 2*row_t
    const int row_t = (lane & 1) + 2 * ((lane >> 2) & 1) + 4 * ((lane >> 3) & 1) + 8 * ((lane >> 4) & 1);
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quarter) << 16);
    float l_part[kV], mr[kV];  // per row of this thread: partial sum and running max
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      l_part[j] = 0.f;
      mr[j] = -INFINITY;
    }
    const int64_t qpos0 = seqlen - p.q_len + j0;  // position of this CTA's first query
    bool ok = true;
    for (int i = 0; i < n_pages; ++i) {
      const int sb = i & 1;
      // A timed-out wait is acted on at the page's one block-wide vote below,
      // where all softmax threads leave together.
      ok = mbar_wait(bar(L::kBarSFull + sb), (uint32_t)((i >> 1) & 1), abort_flag, p.status,
                     p.wait_limit_ns);
      tc_fence_after();
      float sv[kV];
      if constexpr (L::kSplitQ) {
        float lo[16];
        tmem_ld16x64b_x16(t_lane + L::kColS + sb * L::kSCols, sv);
        tmem_ld16x64b_x16(t_lane + L::kColS + sb * L::kSCols + NR, lo);
        tc_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          asm volatile("" : "+f"(sv[k]), "+f"(lo[k]));  // defined only after the wait
          sv[k] += lo[k];
        }
      } else {
#pragma unroll
        for (int c = 0; c < NR / 32; ++c) {
          float tmp[16];
          tmem_ld16x64b_x16(t_lane + L::kColS + sb * NR + 32 * c, tmp);
#pragma unroll
          for (int k = 0; k < 16; ++k) sv[16 * c + k] = tmp[k];
        }
        tc_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar(L::kBarSFree + sb));

      bool exceed = false;
      if ((p_begin + i + 1) * kPage - 1 <= qpos0 && jn == NR / 32) {
        // every token of the page is visible to every row: no mask
#pragma unroll
        for (int j = 0; j < kV; ++j) exceed |= sv[j] > mr[j] + kLazyMax;
      } else {
        const int64_t tpos = (p_begin + i) * kPage + tok;
#pragma unroll
        for (int j = 0; j < kV; ++j) {
          const int jr = j >> 4;  // query of row pr + 2j within this CTA
          const bool vis = jr < jn && tpos <= qpos0 + jr;
          sv[j] = vis ? sv[j] : -INFINITY;
          exceed |= sv[j] > mr[j] + kLazyMax;
        }
      }
      // P buffer i % kPBufs is free once the PV of page i - kPBufs has completed
      bool okp = true;
      if (i >= L::kPBufs) {
        const int pi = i - L::kPBufs;
        okp = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1), abort_flag,
                        p.status, p.wait_limit_ns);
      }
      // one vote per page: nothing to do unless a row's maximum moved or a wait timed out
      if (named_bar_or(1, kSoftmaxThreads, exceed || !ok || !okp)) {
        if (named_bar_or(1, kSoftmaxThreads, !ok || !okp)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < NR / 32; ++c) {
          float tmp[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) tmp[k] = sv[16 * c + k];
          xpose_reduce16<true>(tmp, lane);
          red[quarter * NR + pr + 2 * (16 * c + row_t)] = tmp[0];
        }
        named_bar_sync(1, kSoftmaxThreads);
        if (tid < NR) {
          const float mo = m_used[tid];
          float mn = mo;
#pragma unroll
          for (int q = 0; q < 4; ++q) mn = fmaxf(mn, red[q * NR + tid]);
          m_next[tid] = mn;
          alpha_s[tid] = (mn == -INFINITY) ? 1.f : ex2(mo - mn);
        }
        named_bar_sync(1, kSoftmaxThreads);
        if (i > 0) {
          // rescale the running O^T once every tensor-core update of it has landed
          const int pi = i - 1;
          const bool okw = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1),
                                     abort_flag, p.status, p.wait_limit_ns);
          if (named_bar_or(1, kSoftmaxThreads, !okw)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
#pragma unroll
            for (int c = 0; c < NR / 32; ++c) {
              float o[32];
              const uint32_t ta = t_lane + L::kColO + m * NR + 32 * c;
              tmem_ld32(ta, o);
              tc_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] *= alpha_s[32 * c + k];
              tmem_st32(ta, o);
            }
          }
          tc_wait_st();
        }
#pragma unroll
        for (int j = 0; j < kV; ++j) l_part[j] *= alpha_s[pr + 2 * j];
        if (tid < NR) m_used[tid] = m_next[tid];
        named_bar_sync(1, kSoftmaxThreads);
#pragma unroll
        for (int j = 0; j < kV; ++j) mr[j] = m_used[pr + 2 * j];
      }
      if (p_begin + i == npages - 1 && (seqlen % kPage) != 0) {
        // Rows past the sequence end in its last block hold whatever the pool
        // holds; zero them so 0-probability tokens cannot inject NaN/Inf into O.
        const int r0 = (int)(seqlen % kPage);
        const int units = (kPage - r0) * 8;  // 16-byte units per 64-column chunk
        for (int e = tid; e < 8 * units; e += kSoftmaxThreads) {
          const int chunk = e / units;  // 0..7: latent chunk of the page
          const int u = e % units;
          const int slot = (4 * i + (chunk >> 1)) % L::kLatSlots;
          uint4* dst = reinterpret_cast<uint4*>(smem + L::kOffLat + slot * L::kLatBytes +
                                                (chunk & 1) * 8192 + r0 * 128);
          dst[u] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // probabilities, rounded to bf16 in pairs (one conversion for rows j and
      // kH + j of this thread) and summed in that precision (the rounded values
      // are read back from the bits)
      uint32_t x[kH];
#pragma unroll
      for (int k = 0; k < kH; ++k) {
        const float p0 = sv[k] == -INFINITY ? 0.f : ex2(sv[k] - mr[k]);
        const float p1 = sv[kH + k] == -INFINITY ? 0.f : ex2(sv[kH + k] - mr[kH + k]);
        x[k] = pack_bf16x2(p0, p1);
        l_part[k] += __uint_as_float(x[k] << 16);
        l_part[kH + k] += __uint_as_float(x[k] & 0xffff0000u);
      }
      // The thread pair (t, t^2) holds the two row parities of one token: each
      // takes the partner's half it needs, so that it owns kV consecutive rows
      // (pr 0: rows 0..kV-1 from the low halves, pr 1: the rest from the high
      // halves), then writes its 16-byte units of the token's P^T row
      // (MN-major, swizzled as the PV operand).
      uint32_t w[kH];
#pragma unroll
      for (int k = 0; k < kH; ++k) {
        const uint32_t rcv = __shfl_xor_sync(0xffffffffu, x[k], 2);
        w[k] = pr == 0 ? __byte_perm(x[k], rcv, 0x5410) : __byte_perm(rcv, x[k], 0x7632);
      }
      uint8_t* prow = smem + L::kOffP + (i % L::kPBufs) * L::kPBytes + tok * L::kPRow;
#pragma unroll
      for (int u = 0; u < kH / 4; ++u) {
        const int unit = pr * (kH / 4) + u;
        const int phys = NR == 32 ? (unit ^ ((tok >> 1) & 3)) : (unit ^ (tok & 7));
        *reinterpret_cast<uint4*>(prow + phys * 16) =
            make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::kBarPFull + sb));
    }

    // ---- epilogue: unnormalised O, running max m and sum l of this split
    const int64_t row0 = w.row0;
    bool have = ok && n_pages > 0;
    if (have) {
      const int pi = n_pages - 1;
      const bool okw = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1),
                                 abort_flag, p.status, p.wait_limit_ns);
      have = !named_bar_or(1, kSoftmaxThreads, !okw);
    }
    bool direct = false;
    if constexpr (L::kSplitQ) direct = p.o_hi != nullptr;
    if (have && direct) {
      // one split per unit: normalise here and write the bf16 hi/lo latent
      // output; the row sums come first, their reciprocals go to m_used
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < NR / 32; ++c) {
        float tmp[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) tmp[k] = l_part[16 * c + k];
        xpose_reduce16<false>(tmp, lane);
        red[quarter * NR + pr + 2 * (16 * c + row_t)] = tmp[0];
      }
      named_bar_sync(1, kSoftmaxThreads);
      if (tid < NR) {
        const float l = red[tid] + red[NR + tid] + red[2 * NR + tid] + red[3 * NR + tid];
        m_used[tid] = l > 0.f ? 1.f / l : 0.f;
      }
      named_bar_sync(1, kSoftmaxThreads);
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + 32 * quarter + lane;
#pragma unroll
        for (int c = 0; c < NR / 32; ++c) {
          float o[32];
          tmem_ld32(t_lane + L::kColO + m * NR + 32 * c, o);
          tc_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int n = 32 * c + k;
            if (n < nrows) {
              const float v = o[k] * m_used[n];
              const __nv_bfloat16 hv = __float2bfloat16_rn(v);
              const int64_t off = (row0 + n) * kDLatent + d;
              p.o_hi[off] = hv;
              p.o_lo[off] = __float2bfloat16_rn(v - __bfloat162float(hv));
            }
          }
        }
      }
    } else if (direct) {
      pdl_wait();  // the previous step's W_UV product may still read these rows
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
      for (int e = tid; e < nrows * kDLatent; e += kSoftmaxThreads) {
        p.o_hi[row0 * kDLatent + e] = z;
        p.o_lo[row0 * kDLatent + e] = z;
      }
    } else if (have) {
      tc_fence_after();
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + 32 * quarter + lane;
#pragma unroll
        for (int c = 0; c < NR / 32; ++c) {
          float o[32];
          tmem_ld32(t_lane + L::kColO + m * NR + 32 * c, o);
          tc_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int n = 32 * c + k;
            if (n < nrows) p.part_o[(row0 + n) * kDLatent + d] = o[k];
          }
        }
      }
#pragma unroll
      for (int c = 0; c < NR / 32; ++c) {
        float tmp[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) tmp[k] = l_part[16 * c + k];
        xpose_reduce16<false>(tmp, lane);
        red[quarter * NR + pr + 2 * (16 * c + row_t)] = tmp[0];
      }
      named_bar_sync(1, kSoftmaxThreads);
      if (tid < nrows) {
        const float l = red[tid] + red[NR + tid] + red[2 * NR + tid] + red[3 * NR + tid];
        p.part_ml[(row0 + tid) * 2 + 0] = m_used[tid];
        p.part_ml[(row0 + tid) * 2 + 1] = l;
      }
    } else if (tid < nrows) {
      pdl_wait();  // the previous step's merge may still read this split's m, l
      p.part_ml[(row0 + tid) * 2 + 0] = -INFINITY;
      p.part_ml[(row0 + tid) * 2 + 1] = 0.f;
    }
  }

}

// The sequence, row group and page range of work item `item` (modes
// kWorkSplit and kWorkRanged: split item % nsplit of unit item / nsplit).
template <int kMode>
__device__ __forceinline__ void split_work_item(const DecodeParams& p, int item, int& b, int& g,
                                                int64_t& seqlen, int64_t& npages,
                                                int64_t& p_begin, int64_t& p_end) {
  const int split = item % p.nsplit;
  const int bg = item / p.nsplit;
  g = bg % p.groups;
  b = bg / p.groups;
  seqlen = p.seqlens[b];
  if (seqlen < p.q_len || seqlen > p.max_seqlen) {
    if (threadIdx.x == 0) record_status(p.status, XMLA_ERR_DEVICE_OOB);
    seqlen = 0;
  }
  npages = (seqlen + kPage - 1) / kPage;
  const int64_t p_lo = kMode == kWorkRanged ? min(p.page_lo, npages) : 0;
  const int64_t p_hi = kMode == kWorkRanged ? min(p.page_hi, npages) : npages;
  const int64_t pps = (p_hi - p_lo + p.nsplit - 1) / p.nsplit;
  p_begin = p_lo + (int64_t)split * pps;
  p_end = min(p_hi, p_begin + pps);
}

// The same from entry `item` of the work table (mode kWorkTable); read after
// the preceding kernel, which wrote the table, has completed.
__device__ __forceinline__ void table_work_item(const DecodeParams& p, int item, int& b, int& g,
                                                int64_t& seqlen, int64_t& npages,
                                                int64_t& p_begin, int64_t& p_end) {
  const int4 e = p.work_tab[item];
  if (e.x >= 0 && e.x < p.batch * p.groups) {
    g = e.x % p.groups;
    b = e.x / p.groups;
    seqlen = p.seqlens[b];
    if (seqlen < p.q_len || seqlen > p.max_seqlen) {
      if (threadIdx.x == 0) record_status(p.status, XMLA_ERR_DEVICE_OOB);
      seqlen = 0;
    }
    npages = (seqlen + kPage - 1) / kPage;
    p_begin = min((int64_t)e.y, npages);
    p_end = min((int64_t)e.z, npages);
  }
}

template <int NR, int kMode, bool kSplitQ>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tmap_pool,
                      const __grid_constant__ CUtensorMap tmap_q, const DecodeParams p) {
  using L = DecodeLayout<NR, kSplitQ>;
  extern __shared__ uint8_t smem_raw[];
  uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  base += pad;
  float* m_used = reinterpret_cast<float*>(smem + L::kOffMUsed);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  const int warp = threadIdx.x >> 5;

  // ---- work item
  // with the split query (prompt chunks, short contexts) later queries see more
  // pages: the grid runs them first, so the short work items fill the tail
  const int item = kSplitQ ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  int b = 0, g = 0;
  int64_t seqlen = 0, npages = 0, p_begin = 0, p_end = 0;
  if constexpr (kMode != kWorkTable)
    split_work_item<kMode>(p, item, b, g, seqlen, npages, p_begin, p_end);

  // ---- setup (independent of the previous kernel's results)
  if (threadIdx.x == 0) decode_init_barriers<NR, kSplitQ>(base + L::kOffBars, abort_flag);
  if (warp == 1) {
    tmem_alloc(base + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 32 * kSoftmaxWarp0 && threadIdx.x < 32 * kSoftmaxWarp0 + NR)
    m_used[threadIdx.x - 32 * kSoftmaxWarp0] = -INFINITY;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  if constexpr (kMode == kWorkTable) {
    // the table comes from the kernel launched before this one
    pdl_wait();
    table_work_item(p, item, b, g, seqlen, npages, p_begin, p_end);
  }
  const int j0 = g * (NR / 32);
  const int jn = min(p.q_len - j0, NR / 32);
  // causal: pages past this CTA's last query position hold nothing it may see
  // (a prefill chunk's early queries; at decode sizes this is the last page)
  p_end = min(p_end, (seqlen - p.q_len + j0 + jn - 1) / kPage + 1);
  const int n_pages = (int)max((int64_t)0, p_end - p_begin);
  const int32_t qrow0 = (int32_t)(((int64_t)b * p.q_len + j0) * (L::kSplitQ ? 64 : 32));
  pdl_launch_dependents();

  const DecodePass w{b, j0, jn, n_pages, seqlen, npages, p_begin, (int64_t)item * NR, qrow0};
  decode_pass<NR, kSplitQ>(smem, base, base + L::kOffBars, tmem_base, tmap_pool, tmap_q, p, w);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}


// Split-K attention that chooses the query's precision per sequence, for a
// batch holding short and long sequences at once.  q_ext is in the split
// layout (hi and lo rows).  A sequence of at most kSplitQMaxSeqlen tokens is
// dominated by a few tokens and its output is large, so the ~2^-9 relative
// error of a single bf16 query reaches the output bound there: it is attended
// with the query as hi + lo parts (tmap_q2, 64-row boxes), one pass of 32 rows
// per query of the CTA's row group.  A longer sequence is attended with the hi
// rows alone (tmap_q, 32-row boxes), NR rows in one pass, with the deeper page
// ring.  The partials are laid out as
// mla_decode_kernel<NR, kMode, false> writes them, so the combine is the same.
// Each pass has a barrier set of its own (a finished pass may still have
// tensor-core arrivals in flight on its barriers).
template <int NR>
struct MixedLayout {
  using LL = DecodeLayout<NR, false>;
  using LS = DecodeLayout<32, true>;
  static constexpr int kShortPasses = NR / 32;
  // the short passes' barrier sets: LS's own, then one more per extra pass
  static constexpr uint32_t kOffBars2 = (LS::kBytes + 7u) & ~7u;
  static constexpr uint32_t kShortBytes = kOffBars2 + (kShortPasses - 1) * LS::kNumBars * 8;
  static constexpr uint32_t kTmemCols = LL::kTmemCols > LS::kTmemCols ? LL::kTmemCols
                                                                       : LS::kTmemCols;
  static constexpr uint32_t kBytes = LL::kBytes > kShortBytes ? LL::kBytes : kShortBytes;
  static constexpr uint32_t kSmem = kBytes + 1024;
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

// The passes of a short sequence in the mixed kernel: one per query of the
// CTA's row group, 32 rows each, with the hi/lo query and a barrier set of its
// own.  (Kept inline: compiled out of line, as a call, it put the kernel's long
// pass into a markedly slower code generation -- verify_q4_b8 430 -> 547 us.)
template <int NR>
__device__ __forceinline__ void mixed_short_passes(uint8_t* smem, uint32_t base, uint32_t tmem_base,
                                                const CUtensorMap* tmap_pool,
                                                const CUtensorMap* tmap_q2,
                                                const DecodeParams* pp, int item, int b, int jg,
                                                int64_t seqlen, int64_t npages, int64_t p_begin,
                                                int64_t p_end) {
  using M = MixedLayout<NR>;
  using LS = typename M::LS;
  const DecodeParams& p = *pp;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LS::kOffAbort);
  float* m_used = reinterpret_cast<float*>(smem + LS::kOffMUsed);
#pragma unroll 1
  for (int jj = 0; jj < M::kShortPasses; ++jj) {
    const int j0 = jg + jj;
    if (j0 >= p.q_len) break;
    const uint32_t bars =
        base + (jj == 0 ? LS::kOffBars : M::kOffBars2 + (uint32_t)(jj - 1) * LS::kNumBars * 8u);
    if (threadIdx.x == 0) decode_init_barriers<32, true>(bars, abort_flag);
    if (threadIdx.x >= 32 * kSoftmaxWarp0 && threadIdx.x < 32 * kSoftmaxWarp0 + 32)
      m_used[threadIdx.x - 32 * kSoftmaxWarp0] = -INFINITY;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int64_t pe = min(p_end, (seqlen - p.q_len + j0) / kPage + 1);
    const int n_pages = (int)max((int64_t)0, pe - p_begin);
    const DecodePass w{b, j0, 1, n_pages, seqlen, npages, p_begin, (int64_t)item * NR + 32 * jj,
                       (int32_t)(((int64_t)b * p.q_len + j0) * 64)};
    decode_pass<32, true>(smem, base, bars, tmem_base, *tmap_pool, *tmap_q2, p, w);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
}

template <int NR, int kMode>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    mla_decode_mixed_kernel(const __grid_constant__ CUtensorMap tmap_pool,
                            const __grid_constant__ CUtensorMap tmap_q,
                            const __grid_constant__ CUtensorMap tmap_q2, const DecodeParams p) {
  using M = MixedLayout<NR>;
  using LL = typename M::LL;
  extern __shared__ uint8_t smem_raw[];
  uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  base += pad;
  float* m_used = reinterpret_cast<float*>(smem + LL::kOffMUsed);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + LL::kOffAbort);
  const int warp = threadIdx.x >> 5;
  const int item = (int)blockIdx.x;
  int b = 0, g = 0;
  int64_t seqlen = 0, npages = 0, p_begin = 0, p_end = 0;
  if constexpr (kMode != kWorkTable)
    split_work_item<kMode>(p, item, b, g, seqlen, npages, p_begin, p_end);

  // ---- setup for a long sequence, as in mla_decode_kernel (a short one
  // discards the barriers and sets up its passes in their own layout)
  if (threadIdx.x == 0) decode_init_barriers<NR, false>(base + LL::kOffBars, abort_flag);
  if (warp == 1) {
    tmem_alloc(base + LL::kOffTmem, M::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 32 * kSoftmaxWarp0 && threadIdx.x < 32 * kSoftmaxWarp0 + NR)
    m_used[threadIdx.x - 32 * kSoftmaxWarp0] = -INFINITY;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + LL::kOffTmem);
  if constexpr (kMode == kWorkTable) {
    pdl_wait();  // the table comes from the kernel launched before this one
    table_work_item(p, item, b, g, seqlen, npages, p_begin, p_end);
  }
  const int jg = g * (NR / 32);
  pdl_launch_dependents();
  if (seqlen > kSplitQMaxSeqlen) {
    const int jn = min(p.q_len - jg, NR / 32);
    p_end = min(p_end, (seqlen - p.q_len + jg + jn - 1) / kPage + 1);
    const int n_pages = (int)max((int64_t)0, p_end - p_begin);
    const DecodePass w{b, jg, jn, n_pages, seqlen, npages, p_begin, (int64_t)item * NR,
                       (int32_t)(((int64_t)b * p.q_len + jg) * 64)};
    decode_pass<NR, false, true>(smem, base, base + LL::kOffBars, tmem_base, tmap_pool, tmap_q, p,
                                 w);
  } else {
    __syncthreads();  // every thread holds the tensor-memory base: its slot lies in the short ring
    if (threadIdx.x == 0) {
      for (int i = 0; i < LL::kNumBars; ++i)
        asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(base + LL::kOffBars + 8u * i)
                     : "memory");
    }
    mixed_short_passes<NR>(smem, base, tmem_base, &tmap_pool, &tmap_q2, &p, item, b, jg, seqlen,
                           npages, p_begin, p_end);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, M::kTmemCols);
  }
}

template <int NR, int kMode, bool kSplitQ>
static cudaError_t launch_decode(const CUtensorMap& tp, const CUtensorMap& tq, const DecodeParams& dp,
                                 int64_t items, cudaStream_t st) {
  using L = DecodeLayout<NR, kSplitQ>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(mla_decode_kernel<NR, kMode, kSplitQ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return launch_pdl(mla_decode_kernel<NR, kMode, kSplitQ>, dim3((unsigned)items),
                    dim3(kDecodeThreads), L::kSmem, st, tp, tq, dp);
}


template <int NR, bool kSplitQ>
static cudaError_t launch_mode(int mode, const CUtensorMap& pool_map, const CUtensorMap& q_map,
                               const DecodeParams& dp, int64_t items, cudaStream_t st) {
  if (mode == kWorkTable)
    return launch_decode<NR, kWorkTable, kSplitQ>(pool_map, q_map, dp, items, st);
  if (mode == kWorkRanged)
    return launch_decode<NR, kWorkRanged, kSplitQ>(pool_map, q_map, dp, items, st);
  return launch_decode<NR, kWorkSplit, kSplitQ>(pool_map, q_map, dp, items, st);
}

cudaError_t launch_split_kv(int nr, bool split_q, const CUtensorMap& pool_map,
                            const CUtensorMap& q_map, const DecodeParams& dp, int64_t items,
                            cudaStream_t st) {
  const int mode = dp.work_tab != nullptr                          ? kWorkTable
                   : (dp.page_lo != 0 || dp.page_hi != INT64_MAX) ? kWorkRanged
                                                                  : kWorkSplit;
  if (nr == 32)
    return split_q ? launch_mode<32, true>(mode, pool_map, q_map, dp, items, st)
                   : launch_mode<32, false>(mode, pool_map, q_map, dp, items, st);
  if (nr == 64 && !split_q) return launch_mode<64, false>(mode, pool_map, q_map, dp, items, st);
  return cudaErrorInvalidValue;
}


template <int NR, int kMode>
static cudaError_t launch_mixed(const CUtensorMap& tp, const CUtensorMap& tq,
                                const CUtensorMap& tq2, const DecodeParams& dp, int64_t items,
                                cudaStream_t st) {
  using M = MixedLayout<NR>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(mla_decode_mixed_kernel<NR, kMode>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, M::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return launch_pdl(mla_decode_mixed_kernel<NR, kMode>, dim3((unsigned)items),
                    dim3(kDecodeThreads), M::kSmem, st, tp, tq, tq2, dp);
}

cudaError_t launch_split_kv_mixed(int nr, const CUtensorMap& pool_map, const CUtensorMap& q_map,
                                  const CUtensorMap& q2_map, const DecodeParams& dp,
                                  int64_t items, cudaStream_t st) {
  const int mode = dp.work_tab != nullptr                          ? kWorkTable
                   : (dp.page_lo != 0 || dp.page_hi != INT64_MAX) ? kWorkRanged
                                                                  : kWorkSplit;
  if (nr != 32 && nr != 64) return cudaErrorInvalidValue;
  if (mode == kWorkTable)
    return nr == 32 ? launch_mixed<32, kWorkTable>(pool_map, q_map, q2_map, dp, items, st)
                    : launch_mixed<64, kWorkTable>(pool_map, q_map, q2_map, dp, items, st);
  if (mode == kWorkRanged)
    return nr == 32 ? launch_mixed<32, kWorkRanged>(pool_map, q_map, q2_map, dp, items, st)
                    : launch_mixed<64, kWorkRanged>(pool_map, q_map, q2_map, dp, items, st);
  return nr == 32 ? launch_mixed<32, kWorkSplit>(pool_map, q_map, q2_map, dp, items, st)
                  : launch_mixed<64, kWorkSplit>(pool_map, q_map, q2_map, dp, items, st);
}

}  // namespace xmla
