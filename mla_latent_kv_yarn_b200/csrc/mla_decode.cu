// MLA decode over the paged latent cache, weight-absorbed form.
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
// Three kernels per call, chained with programmatic dependent launch:
//   q_absorb   q_ext[b,j,h] = c * [W_UK[h]^T q_nope | rope(q_pe)]   (c = scale * log2 e)
//   decode     one CTA per (sequence, row group, KV split): 64-token pages are
//              streamed by TMA into a shared-memory ring; S^T = page . q_ext^T
//              (M = 64 tokens, N = rows, K = 576) and O^T += c_kv^T . P^T (M = 128
//              latent dims x 4, N = rows, K = 64 tokens) run on tcgen05 with fp32
//              accumulators in tensor memory; S is double-buffered so the QK of
//              page i+1 runs while the softmax of page i does; the online softmax
//              (base 2, lazy max update) runs in registers.  Writes per-split
//              (m, l, O).
//   combine    a cluster of 8 CTAs per (head, row chunk) merges the splits by their
//              log-sum-exp over 64-dim slices of the latent and applies W_UV; the
//              slices' partial outputs are summed through distributed shared memory.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "xmla_device.cuh"
#include "yarn.cuh"

namespace cg = cooperative_groups;

namespace xmla {

constexpr float kLog2e = 1.4426950408889634f;
// A row's running maximum is only raised when a score exceeds it by more than
// this (log2 units), so probabilities stay <= 2^kLazyMax before normalisation.
constexpr float kLazyMax = 8.0f;
constexpr int kMaxSplits = 1024;
constexpr int kSoftmaxThreads = 128;
constexpr int kSoftmaxWarp0 = 3;  // warps: 0 TMA producer, 1 QK issuer, 2 PV issuer, 3-6 softmax
constexpr int kDecodeThreads = 32 * kSoftmaxWarp0 + kSoftmaxThreads;

// ---------------------------------------------------------------- shared-memory plan

template <int NR>
struct DecodeLayout {
  static_assert(NR == 32 || NR == 64, "rows per CTA");
  static constexpr int kLatSlots = NR == 32 ? 9 : 7;   // 16 KB: latent dims 128m..128m+127 of a page
  static constexpr int kRopeSlots = NR == 32 ? 4 : 2;  // 8 KB: rope dims of a page
  static constexpr uint32_t kQChunk = NR * 128;        // one 64-column chunk of q_ext
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
  static constexpr uint32_t kOffLat = kOffP + 2 * kPBytes;
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
  // tensor memory columns: O^T at [0, 4 NR), S^T buffers at [4 NR, 5 NR) and [5 NR, 6 NR)
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = 4 * NR;
  static constexpr uint32_t kTmemCols = 6 * NR <= 256 ? 256 : 512;
};

struct DecodeParams {
  const int32_t* block_table;
  const int32_t* seqlens;
  float* part_o;   // [items, NR, 512]
  float* part_ml;  // [items, NR, 2]
  int32_t* status;
  int64_t num_blocks;
  int64_t max_seqlen;
  uint64_t wait_limit_ns;
  int32_t max_blocks;
  int32_t batch;
  int32_t q_len;
  int32_t groups;
  int32_t nsplit;
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

template <int NR>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tmap_pool,
                      const __grid_constant__ CUtensorMap tmap_q, const DecodeParams p) {
  using L = DecodeLayout<NR>;
  extern __shared__ uint8_t smem_raw[];
  uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  base += pad;

  auto bar = [&](int i) -> uint32_t { return base + L::kOffBars + 8u * (uint32_t)i; };
  float* m_used = reinterpret_cast<float*>(smem + L::kOffMUsed);
  float* m_next = reinterpret_cast<float*>(smem + L::kOffMNext);
  float* alpha_s = reinterpret_cast<float*>(smem + L::kOffAlpha);
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item
  const int item = blockIdx.x;
  const int split = item % p.nsplit;
  const int bg = item / p.nsplit;
  const int g = bg % p.groups;
  const int b = bg / p.groups;
  const int j0 = g * (NR / 32);
  const int jn = min(p.q_len - j0, NR / 32);
  const int nrows = jn * 32;
  int64_t seqlen = p.seqlens[b];
  if (seqlen < p.q_len || seqlen > p.max_seqlen) {
    if (threadIdx.x == 0) record_status(p.status, XMLA_ERR_DEVICE_OOB);
    seqlen = 0;
  }
  const int64_t npages = (seqlen + kPage - 1) / kPage;
  const int64_t pps = (npages + p.nsplit - 1) / p.nsplit;
  const int64_t p_begin = (int64_t)split * pps;
  const int64_t p_end = min(npages, p_begin + pps);
  const int n_pages = (int)max((int64_t)0, p_end - p_begin);

  // ---- setup (independent of the previous kernel's results)
  if (threadIdx.x == 0) {
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
  const int32_t qrow0 = (int32_t)(((int64_t)b * p.q_len + j0) * 32);
  pdl_launch_dependents();

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0 && n_pages > 0) {
      tma_prefetch_desc(&tmap_pool);
      tma_prefetch_desc(&tmap_q);
      const uint64_t stream_policy = policy_evict_first();
      int li = 0, ri = 0;
      uint32_t lph = 0, rph = 0;
      int64_t lat_issued = 0, rope_issued = 0;
      bool ok = true, q_issued = false;
      // block ids are fetched four pages ahead so their load latency is hidden
      const int32_t* bt = p.block_table + (int64_t)b * p.max_blocks + p_begin;
      int32_t nb0 = bt[0];
      int32_t nb1 = n_pages > 1 ? bt[1] : 0;
      int32_t nb2 = n_pages > 2 ? bt[2] : 0;
      int32_t nb3 = n_pages > 3 ? bt[3] : 0;
      const int64_t first_new = seqlen - p.q_len;  // first row appended by this step
      bool waited = false;
      for (int i = 0; i < n_pages && ok; ++i) {
        if (!waited && (p_begin + i + 1) * kPage > first_new) {
          // this page holds rows written by the kernels launched just before:
          // wait for them (through q_absorb's completion) before reading it
          pdl_wait();
          waited = true;
        }
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
        if (!mbar_wait(bar(L::kBarRopeEmpty + ri), rph ^ 1u, abort_flag, p.status,
                       p.wait_limit_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::kBarRopeFull + ri), L::kRopeBytes);
        tma_load_2d_hint(base + L::kOffRope + ri * L::kRopeBytes, &tmap_pool, kDLatent, y,
                         bar(L::kBarRopeFull + ri), stream_policy);
        ++rope_issued;
        if (++ri == L::kRopeSlots) { ri = 0; rph ^= 1u; }
        if (!q_issued) {
          // q_ext is the previous kernel's output: wait for it only after the
          // first page is on its way.
          if (!waited) pdl_wait();
          waited = true;
          mbar_arrive_expect_tx(bar(L::kBarQ), 9u * L::kQChunk);
          for (int c = 0; c < 9; ++c)
            tma_load_2d(base + L::kOffQ + c * L::kQChunk, &tmap_q, c * 64, qrow0, bar(L::kBarQ));
          q_issued = true;
        }
      }
      // Every copy issued must land before the CTA may exit: wait for the last
      // phase armed on each slot (immediate when the consumer already saw it).
      if (q_issued) mbar_wait(bar(L::kBarQ), 0, nullptr, p.status, p.wait_limit_ns);
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
      constexpr uint32_t idesc_qk = idesc_bf16_f32(64, NR, false, false);
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
          const uint32_t t_s = tmem_base + L::kColS + sb * NR;
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
                            (m | half | k) != 0 ? 1u : 0u);
            }
          }
          if (!ok) break;
          const int r = i % L::kRopeSlots;
          if (!(ok = wait(L::kBarRopeFull + r, (uint32_t)((i / L::kRopeSlots) & 1)))) break;
          tc_fence_after();
          const uint64_t ar = d_rope_k + ((r * L::kRopeBytes) >> 4);
          const uint64_t bq = d_q + ((8 * L::kQChunk) >> 4);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_bf16(t_s, ar + ((k * 32) >> 4), bq + ((k * 32) >> 4), idesc_qk, 1u);
          tc_commit(bar(L::kBarSFull + sb));
          tc_commit(bar(L::kBarRopeEmpty + r));
        }
      } else {
        for (int i = 0; i < n_pages && ok; ++i) {
          if (!(ok = wait(L::kBarPFull + (i & 1), (uint32_t)((i >> 1) & 1)))) break;
          tc_fence_after();
          const uint64_t bp = d_p + (((i & 1) * L::kPBytes) >> 4);
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
      ok = mbar_wait(bar(L::kBarSFull + sb), (uint32_t)((i >> 1) & 1), abort_flag, p.status,
                     p.wait_limit_ns);
      if (named_bar_or(1, kSoftmaxThreads, !ok)) { ok = false; break; }
      tc_fence_after();
      float sv[kV];
#pragma unroll
      for (int c = 0; c < NR / 32; ++c) {
        float tmp[16];
        tmem_ld16x64b_x16(t_lane + L::kColS + sb * NR + 32 * c, tmp);
#pragma unroll
        for (int k = 0; k < 16; ++k) sv[16 * c + k] = tmp[k];
      }
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::kBarSFree + sb));

      const int64_t tpos = (p_begin + i) * kPage + tok;
      bool exceed = false;
#pragma unroll
      for (int j = 0; j < kV; ++j) {
        const int jr = j >> 4;  // query of row pr + 2j within this CTA
        const bool vis = jr < jn && tpos <= qpos0 + jr;
        sv[j] = vis ? sv[j] : -INFINITY;
        exceed |= sv[j] > mr[j] + kLazyMax;
      }
      if (named_bar_or(1, kSoftmaxThreads, exceed)) {
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
      if (i >= 2) {
        // P buffer (i & 1) is free once the PV of page i - 2 has completed
        const int pi = i - 2;
        const bool okw = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1),
                                   abort_flag, p.status, p.wait_limit_ns);
        if (named_bar_or(1, kSoftmaxThreads, !okw)) { ok = false; break; }
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
      // probabilities (bf16-rounded, also summed in that precision)
      float pb[kV];
#pragma unroll
      for (int j = 0; j < kV; ++j) {
        const float pf = sv[j] == -INFINITY ? 0.f : ex2(sv[j] - mr[j]);
        pb[j] = __bfloat162float(__float2bfloat16_rn(pf));
        l_part[j] += pb[j];
      }
      // The thread pair (t, t^2) holds the two row parities of one token: swap
      // halves so that each owns kV consecutive rows, then write its 16-byte
      // units of the token's P^T row (MN-major, swizzled as the PV operand).
      uint32_t w[kH];
#pragma unroll
      for (int k = 0; k < kH; ++k) {
        const float own = pr == 0 ? pb[k] : pb[kH + k];
        const float snd = pr == 0 ? pb[kH + k] : pb[k];
        const float rcv = __shfl_xor_sync(0xffffffffu, snd, 2);
        w[k] = pr == 0 ? pack_bf16x2(own, rcv) : pack_bf16x2(rcv, own);
      }
      uint8_t* prow = smem + L::kOffP + sb * L::kPBytes + tok * L::kPRow;
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
    const int64_t row0 = (int64_t)item * NR;
    bool have = ok && n_pages > 0;
    if (have) {
      const int pi = n_pages - 1;
      const bool okw = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1),
                                 abort_flag, p.status, p.wait_limit_ns);
      have = !named_bar_or(1, kSoftmaxThreads, !okw);
    }
    if (have) {
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
      p.part_ml[(row0 + tid) * 2 + 0] = -INFINITY;
      p.part_ml[(row0 + tid) * 2 + 1] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ---------------------------------------------------------------- q absorb

// q_ext[r, h] = qscale * [W_UK[h]^T q_nope[r, h] | rope(q_pe[r, h], pos_r)], r = b*q_len + j,
// with pos_r = seqlens[b] - q_len + j (the q_len new tokens are the last cache
// entries).  grid (32 heads, 8 blocks of 64 latent columns); 128 threads:
// thread t owns 8 columns (t % 8) and 8 of the 128 nope dims (t / 8), holding
// its 8 x 8 slice of W_UK in registers (loaded before the wait on the kernel
// launched just before, which it does not depend on); partial sums meet in
// shared memory.  A ninth block per head rotates the rope part.
constexpr int kAbsorbRows = 8;

// q and seqlens carry no __restrict__ so that their loads stay behind the
// griddepcontrol.wait (a preceding kernel may have written them).
__global__ void __launch_bounds__(128) q_absorb_kernel(const __nv_bfloat16* q,
                                                       const __nv_bfloat16* __restrict__ W_UK,
                                                       const int32_t* seqlens,
                                                       __nv_bfloat16* __restrict__ q_ext, int rows,
                                                       int q_len, float qscale,
                                                       const RopeTable tab) {
  __shared__ float sq[kAbsorbRows][kDNope];
  __shared__ float part[16][kAbsorbRows][64];
  pdl_launch_dependents();
  const int h = blockIdx.x;
  const int cb = blockIdx.y;
  const int t = threadIdx.x;
  if (cb == kDLatent / 64) {
    // q and the cache rows of this step may come from the kernels launched just
    // before; every CTA waits (the decode kernel relies on it, see its producer)
    pdl_wait();
    constexpr int kPairs = kDRope / 2;
    for (int e = t; e < rows * kPairs; e += blockDim.x) {
      const int r = e / kPairs, i = e % kPairs;
      const int64_t pos = (int64_t)seqlens[r / q_len] - q_len + (r % q_len);
      const __nv_bfloat16* x = q + ((int64_t)r * kHeads + h) * kDQ + kDNope;
      double y1, y2;
      rope_pair((double)__bfloat162float(x[i]), (double)__bfloat162float(x[i + kPairs]), pos, i,
                tab, &y1, &y2);
      __nv_bfloat16* o = q_ext + ((int64_t)r * kHeads + h) * kDRow + kDLatent;
      o[i] = __double2bfloat16(y1 * (double)qscale);
      o[i + kPairs] = __double2bfloat16(y2 * (double)qscale);
    }
    return;
  }
  const int c8 = t & 7;
  const int dg = t >> 3;
  float w[8][8];
#pragma unroll
  for (int dd = 0; dd < 8; ++dd) {
    const uint4 v = *reinterpret_cast<const uint4*>(
        W_UK + ((int64_t)h * kDNope + dg * 8 + dd) * kDLatent + cb * 64 + c8 * 8);
    const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      w[dd][2 * e] = __low2float(pv[e]);
      w[dd][2 * e + 1] = __high2float(pv[e]);
    }
  }
  pdl_wait();
  for (int r0 = 0; r0 < rows; r0 += kAbsorbRows) {
    const int nr = min(kAbsorbRows, rows - r0);
    __syncthreads();
    for (int e = t; e < nr * kDNope; e += blockDim.x) {
      const int r = e / kDNope, d = e % kDNope;
      sq[r][d] = __bfloat162float(q[((int64_t)(r0 + r) * kHeads + h) * kDQ + d]);
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int dd = 0; dd < 8; ++dd) {
        const float x = sq[r][dg * 8 + dd];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = fmaf(x, w[dd][k], acc[k]);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) part[dg][r][c8 * 8 + k] = acc[k];
    }
    __syncthreads();
    for (int o = t; o < nr * 64; o += blockDim.x) {
      const int r = o / 64, col = o % 64;
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) s += part[k][r][col];
      q_ext[((int64_t)(r0 + r) * kHeads + h) * kDRow + cb * 64 + col] = __float2bfloat16_rn(s * qscale);
    }
  }
}

// ---------------------------------------------------------------- combine + W_UV

// Cluster of 8 CTAs per (head h, chunk of up to kCombineRows output rows).
// CTA `slice` owns latent dims [64 slice, 64 slice + 64).  All rows of the
// chunk are merged together: 16 groups of 16 threads (one float4 of the slice
// each) are shared out over the rows, and a row's splits are dealt round-robin
// over its groups, so one pass of loads covers the chunk.  Every split is
// weighted by 2^(m_s - M) against the row's overall maximum M and the sum is
// divided by L = sum_s l_s 2^(m_s - M).  The CTA then multiplies its merged
// 64 dims by the matching 64 rows of W_UV[h] and sends each 16-column block of
// that product to the CTA that owns the block (distributed shared memory); the
// owner adds the 8 contributions and writes its 16 output columns.
constexpr int kSlices = 8;
constexpr int kSliceDims = kDLatent / kSlices;        // 64
constexpr int kCombineRows = 16;
constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombineGroups = kCombineThreads / 16;  // 16 threads x float4 cover a split row's slice
constexpr int kCombineDepth = 10;                     // split rows each thread keeps in flight
constexpr int kStatDepth = 4;                         // (m, l) pairs each lane keeps in flight
constexpr int kColsPerSlice = kDV / kSlices;          // 16

// Online (max, sum-of-exp2) pair merge.
__device__ __forceinline__ void lse_merge(float& m, float& l, float m2, float l2) {
  const float mx = fmaxf(m, m2);
  if (mx == -INFINITY) return;
  l = l * ex2(m - mx) + l2 * ex2(m2 - mx);
  m = mx;
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__global__ void __cluster_dims__(kSlices, 1, 1) __launch_bounds__(kCombineThreads, 3)
    combine_uv_kernel(const float* part_o, const float* part_ml,
                      const __nv_bfloat16* __restrict__ W_UV, __nv_bfloat16* __restrict__ out,
                      int rows, int q_len, int groups, int nsplit, int rows_per_cta) {
  // part_o and part_ml are written by the kernel launched just before this one,
  // which lets this grid start early: they carry no __restrict__, so their loads
  // are not taken as invariant and stay behind the griddepcontrol.wait below.
  __shared__ __align__(16) __nv_bfloat16 w_s[kSliceDims][kDV];  // this slice's rows of W_UV[h]
  __shared__ __align__(16) float4 acc_s[kCombineGroups][kSliceDims / 4];
  __shared__ __align__(16) float o_s[kCombineRows][kSliceDims];
  __shared__ __align__(16) float inbox[kSlices][kCombineRows][kColsPerSlice];  // by sender slice
  __shared__ float stat_m[kCombineRows][kCombineWarps], stat_l[kCombineRows][kCombineWarps];
  cg::cluster_group cluster = cg::this_cluster();
  const int slice = (int)cluster.block_rank();
  const int cid = blockIdx.x / kSlices;
  const int h = cid % kHeads;
  const int chunk = cid / kHeads;
  const int r0 = chunk * kCombineRows;
  const int nr = min(kCombineRows, rows - r0);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  pdl_launch_dependents();
  // first half of the barrier that guarantees every CTA of the cluster runs
  // before any of them writes into another's shared memory
  cluster_arrive_relaxed();
  // W_UV does not depend on the decode kernel: stage it while that kernel finishes
  {
    const uint4* src = reinterpret_cast<const uint4*>(W_UV + ((int64_t)h * kDLatent + slice * kSliceDims) * kDV);
    uint4* dst = reinterpret_cast<uint4*>(&w_s[0][0]);
#pragma unroll
    for (int e = 0; e < kSliceDims * kDV / 8 / kCombineThreads; ++e)
      dst[tid + kCombineThreads * e] = src[tid + kCombineThreads * e];
  }

  // partial row of split 0 for chunk row rr; split s is s * rows_per_cta rows further
  auto split0_row = [&](int rr) -> int64_t {
    const int r = r0 + rr;  // r = b*q_len + j
    const int b = r / q_len, j = r % q_len;
    const int ridx = j * kHeads + h;
    return ((int64_t)b * groups + ridx / rows_per_cta) * nsplit * rows_per_cta + ridx % rows_per_cta;
  };
  const int q4 = tid & 15;  // float4 of the 64-dim slice
  const int grp = tid >> 4;
  const int gpr = max(1, kCombineGroups / nr);  // groups per row
  const int my_rr = grp / gpr;
  const int sub = grp % gpr;
  const bool active = my_rr < nr;
  const int64_t base = active ? split0_row(my_rr) : 0;
  const float* po = part_o + base * kDLatent + slice * kSliceDims + 4 * q4;
  const float* pm = part_ml + 2 * base;          // m of split s at pm[s * m_stride]
  const int o_stride = rows_per_cta * kDLatent;  // floats between splits (nsplit * o_stride < 2^31)
  const int m_stride = 2 * rows_per_cta;
  const int wpr = max(1, kCombineWarps / nr);    // warps per row for the statistics

  pdl_wait();  // the split partials come from the decode kernel

  // first batch of this thread's split rows, issued before the row statistics
  // so that both sets of loads are in flight together.  A split that saw no
  // token has m = -inf (and l = 0); only m is needed to recognise it.
  float4 v[kCombineDepth];
  float ms[kCombineDepth];
#pragma unroll
  for (int k = 0; k < kCombineDepth; ++k) {
    const int s = sub + gpr * k;
    const bool in = active && s < nsplit;
    v[k] = in ? *reinterpret_cast<const float4*>(po + s * o_stride) : make_float4(0.f, 0.f, 0.f, 0.f);
    ms[k] = in ? pm[s * m_stride] : -INFINITY;
  }

  // row statistics: `wpr` warps share a row's splits (part p takes splits
  // 32 p + lane, then every 32 wpr further); each warp reduces its share
  {
    const int part = warp % wpr;
    for (int rr = warp / wpr; rr < nr; rr += kCombineWarps / wpr) {
      const float2* rml = reinterpret_cast<const float2*>(part_ml) + split0_row(rr);
      float m = -INFINITY, l = 0.f;
      for (int s0 = 32 * part; s0 < nsplit; s0 += 32 * wpr * kStatDepth) {
        float2 x[kStatDepth];
#pragma unroll
        for (int k = 0; k < kStatDepth; ++k) {
          const int s = s0 + lane + 32 * wpr * k;
          x[k] = s < nsplit ? rml[(int64_t)s * rows_per_cta] : make_float2(-INFINITY, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kStatDepth; ++k)
          if (x[k].y > 0.f) lse_merge(m, l, x[k].x, x[k].y);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
        lse_merge(m, l, m2, l2);
      }
      if (lane == 0) {
        stat_m[rr][part] = m;
        stat_l[rr][part] = l;
      }
    }
  }
  __syncthreads();

  // weighted sum of this thread's split rows (the partial O of a split that saw
  // no token was never written: it is skipped, not multiplied by zero)
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) {
    float M = stat_m[my_rr][0];
    for (int p = 1; p < wpr; ++p) M = fmaxf(M, stat_m[my_rr][p]);
    for (int k0 = 0;; k0 += kCombineDepth) {
#pragma unroll
      for (int k = 0; k < kCombineDepth; ++k) {
        if (ms[k] != -INFINITY) {
          const float wgt = ex2(ms[k] - M);
          acc.x = fmaf(wgt, v[k].x, acc.x);
          acc.y = fmaf(wgt, v[k].y, acc.y);
          acc.z = fmaf(wgt, v[k].z, acc.z);
          acc.w = fmaf(wgt, v[k].w, acc.w);
        }
      }
      const int k1 = k0 + kCombineDepth;
      if (sub + gpr * k1 >= nsplit) break;
#pragma unroll
      for (int k = 0; k < kCombineDepth; ++k) {
        const int s = sub + gpr * (k1 + k);
        const bool in = s < nsplit;
        v[k] = in ? *reinterpret_cast<const float4*>(po + s * o_stride) : make_float4(0.f, 0.f, 0.f, 0.f);
        ms[k] = in ? pm[s * m_stride] : -INFINITY;
      }
    }
  }
  acc_s[grp][q4] = acc;
  __syncthreads();
  for (int e = tid; e < nr * kSliceDims; e += kCombineThreads) {
    const int rr = e / kSliceDims, d = e % kSliceDims;
    float M = stat_m[rr][0];
    for (int p = 1; p < wpr; ++p) M = fmaxf(M, stat_m[rr][p]);
    float L = 0.f;
    for (int p = 0; p < wpr; ++p)
      if (stat_l[rr][p] > 0.f) L += stat_l[rr][p] * ex2(stat_m[rr][p] - M);
    const float* a = reinterpret_cast<const float*>(&acc_s[rr * gpr][0]) + d;
    float t = 0.f;
    for (int g = 0; g < gpr; ++g) t += a[g * kSliceDims];
    o_s[rr][d] = L > 0.f ? t / L : 0.f;
  }
  __syncthreads();

  // slice product: sum over the slice's 64 latent dims c of o[r][c] W_UV[h][c][v]
  // for the column pair (2 vp, 2 vp + 1), sent to the CTA owning that column block
  cluster_wait_acquire();  // every CTA of the cluster is running
  {
    const int vp = tid & (kDV / 2 - 1);
    const int owner = (2 * vp) / kColsPerSlice;
    float* dst = cluster.map_shared_rank(&inbox[slice][0][0], owner);
    for (int rr = tid / (kDV / 2); rr < nr; rr += kCombineThreads / (kDV / 2)) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 16
      for (int c = 0; c < kSliceDims; ++c) {
        const float2 w = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(&w_s[c][0])[vp]);
        const float x = o_s[rr][c];
        a0 = fmaf(x, w.x, a0);
        a1 = fmaf(x, w.y, a1);
      }
      *reinterpret_cast<float2*>(dst + rr * kColsPerSlice + (2 * vp) % kColsPerSlice) = make_float2(a0, a1);
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();  // all 8 contributions have landed in this CTA's inbox
  if (tid < nr * kColsPerSlice) {
    const int rr = tid / kColsPerSlice, c = tid % kColsPerSlice;
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < kSlices; ++k) t += inbox[k][rr][c];
    out[((int64_t)(r0 + rr) * kHeads + h) * kDV + slice * kColsPerSlice + c] = __float2bfloat16_rn(t);
  }
}

// ---------------------------------------------------------------- self-test kernel

__global__ void wait_timeout_selftest_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar_word;
  const uint32_t b = smem_u32(&bar_word);
  mbar_init(b, 1);
  fence_barrier_init();
  // nothing ever arrives on this barrier: the bounded wait must give up
  mbar_wait(b, 0, nullptr, status, limit_ns);
}

// ---------------------------------------------------------------- host plan

struct Plan {
  int nr;       // rows per CTA (32 or 64)
  int groups;   // row groups per sequence
  int nsplit;   // KV splits per (sequence, group)
  int64_t items;
  size_t off_qext, off_o, off_ml, bytes;
};

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static bool make_plan(int32_t B, int32_t q_len, int64_t max_seqlen, int32_t num_sms,
                      int32_t num_splits, Plan* pl) {
  if (B < 1 || q_len < 1 || q_len > kMaxQLen || max_seqlen < q_len ||
      max_seqlen > (int64_t)0x7fffffff - kPage || num_sms < 1 || num_splits < 0)
    return false;
  Plan P;
  P.nr = q_len == 1 ? 32 : 64;
  P.groups = (q_len * 32 + P.nr - 1) / P.nr;
  const int64_t max_pages = (max_seqlen + kPage - 1) / kPage;
  int64_t ns;
  if (num_splits > 0) {
    ns = num_splits;
  } else {
    const int64_t units = (int64_t)B * P.groups;
    ns = units >= num_sms ? 1 : num_sms / units;
    const int64_t cap = max_pages >= 2 ? max_pages / 2 : 1;  // at least two pages per split
    if (ns > cap) ns = cap;
  }
  if (ns < 1) ns = 1;
  if (ns > kMaxSplits) return false;
  P.nsplit = (int)ns;
  P.items = (int64_t)B * P.groups * P.nsplit;
  if (P.items > 0x7fffffff) return false;
  const size_t qext = (size_t)B * q_len * kHeads * kDRow * 2;
  P.off_qext = 0;
  P.off_o = align_up(qext, 1024);
  P.off_ml = align_up(P.off_o + (size_t)P.items * P.nr * kDLatent * 4, 1024);
  P.bytes = align_up(P.off_ml + (size_t)P.items * P.nr * 2 * 4, 1024);
  *pl = P;
  return true;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D map over rows of 576 bf16 (1152 B), box = 64 columns x box_rows rows,
// 128-byte swizzle (the layout the tensor-core descriptors above expect).
static bool encode_rows576(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDRow, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDRow * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NR>
static cudaError_t launch_decode(const CUtensorMap& tp, const CUtensorMap& tq, const DecodeParams& dp,
                                 int64_t items, cudaStream_t st) {
  using L = DecodeLayout<NR>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(mla_decode_kernel<NR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return launch_pdl(mla_decode_kernel<NR>, dim3((unsigned)items), dim3(kDecodeThreads), L::kSmem,
                    st, tp, tq, dp);
}

static bool device_ok(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev);
  return major == 10 && minor == 0;
}

}  // namespace xmla

using namespace xmla;

extern "C" size_t xmla_decode_workspace_size(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                             int32_t num_sms, int32_t num_splits) {
  Plan P;
  return make_plan(batch, q_len, max_seqlen, num_sms, num_splits, &P) ? P.bytes : 0;
}

extern "C" int32_t xmla_decode_num_splits(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                          int32_t num_sms, int32_t num_splits) {
  Plan P;
  return make_plan(batch, q_len, max_seqlen, num_sms, num_splits, &P) ? P.nsplit : 0;
}

static cudaError_t record_event(void* ev, cudaStream_t st) {
  if (ev == nullptr) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  // inside a graph capture the record must become an event-record node
  return cs == cudaStreamCaptureStatusActive
             ? cudaEventRecordWithFlags((cudaEvent_t)ev, st, cudaEventRecordExternal)
             : cudaEventRecord((cudaEvent_t)ev, st);
}

extern "C" xmla_status xmla_decode_profiled(const xmla_yarn_cfg* cfg, const void* q,
                                            const void* W_UK, const void* W_UV,
                                            const void* pool, int64_t num_blocks,
                                            const int32_t* block_table, int32_t max_blocks,
                                            const int32_t* seqlens, int32_t batch, int32_t q_len,
                                            int64_t max_seqlen, float softmax_scale,
                                            int32_t num_splits, void* workspace,
                                            size_t workspace_bytes, int32_t* status_dev, void* out,
                                            void* stream, void* attn_start, void* attn_stop) {
  if (q == nullptr || W_UK == nullptr || W_UV == nullptr || pool == nullptr ||
      block_table == nullptr || seqlens == nullptr || workspace == nullptr || out == nullptr)
    return XMLA_ERR_INVALID_ARG;
  if (!yarn_cfg_ok(cfg)) return XMLA_ERR_INVALID_ARG;
  if (cfg->rotary_dim != kDRope) return XMLA_ERR_SHAPE;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return XMLA_ERR_INVALID_ARG;
  if ((((uintptr_t)pool) & 15u) || (((uintptr_t)workspace) & 255u) || (((uintptr_t)q) & 15u) ||
      (((uintptr_t)W_UK) & 15u) || (((uintptr_t)W_UV) & 15u) || (((uintptr_t)out) & 15u))
    return XMLA_ERR_INVALID_ARG;
  if (num_blocks < 1 || num_blocks * kPage >= 0x7fffffffLL || max_blocks < 1 ||
      (int64_t)max_blocks * kPage < max_seqlen)
    return XMLA_ERR_SHAPE;
  int nsm = 0;
  if (!device_ok(&nsm)) return XMLA_ERR_UNSUPPORTED;
  Plan P;
  if (!make_plan(batch, q_len, max_seqlen, nsm, num_splits, &P)) return XMLA_ERR_SHAPE;
  if (workspace_bytes < P.bytes) return XMLA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* ws = (uint8_t*)workspace;
  __nv_bfloat16* q_ext = (__nv_bfloat16*)(ws + P.off_qext);
  const int rows = batch * q_len;

  CUtensorMap tmap_pool, tmap_q;
  if (!encode_rows576(&tmap_pool, pool, (uint64_t)num_blocks * kPage, kPage)) return XMLA_ERR_CUDA;
  if (!encode_rows576(&tmap_q, q_ext, (uint64_t)rows * kHeads, (uint32_t)P.nr)) return XMLA_ERR_CUDA;

  const float qscale = softmax_scale * kLog2e;
  // Every kernel of the chain waits (griddepcontrol.wait) for its predecessor
  // before reading anything a kernel of this step may have written, so once
  // q_absorb completes all earlier work on the stream has landed.
  if (launch_pdl(q_absorb_kernel, dim3(kHeads, kDLatent / 64 + 1), dim3(128), 0, st,
                 (const __nv_bfloat16*)q, (const __nv_bfloat16*)W_UK, seqlens, q_ext, rows, q_len,
                 qscale, make_rope_table(cfg)) != cudaSuccess)
    return XMLA_ERR_CUDA;

  DecodeParams dp;
  dp.block_table = block_table;
  dp.seqlens = seqlens;
  dp.part_o = (float*)(ws + P.off_o);
  dp.part_ml = (float*)(ws + P.off_ml);
  dp.status = status_dev;
  dp.num_blocks = num_blocks;
  dp.max_seqlen = max_seqlen;
  dp.wait_limit_ns = kWaitLimitNs;
  dp.max_blocks = max_blocks;
  dp.batch = batch;
  dp.q_len = q_len;
  dp.groups = P.groups;
  dp.nsplit = P.nsplit;
  if (record_event(attn_start, st) != cudaSuccess) return XMLA_ERR_CUDA;
  cudaError_t e = P.nr == 32 ? launch_decode<32>(tmap_pool, tmap_q, dp, P.items, st)
                             : launch_decode<64>(tmap_pool, tmap_q, dp, P.items, st);
  if (e != cudaSuccess) return XMLA_ERR_CUDA;
  if (record_event(attn_stop, st) != cudaSuccess) return XMLA_ERR_CUDA;

  const int chunks = (rows + kCombineRows - 1) / kCombineRows;
  e = launch_pdl(combine_uv_kernel, dim3(kSlices * kHeads * chunks), dim3(kCombineThreads), 0, st,
                 (const float*)dp.part_o, (const float*)dp.part_ml, (const __nv_bfloat16*)W_UV,
                 (__nv_bfloat16*)out, rows, q_len, P.groups, P.nsplit, P.nr);
  return e == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}

extern "C" xmla_status xmla_decode(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                   const void* W_UV, const void* pool, int64_t num_blocks,
                                   const int32_t* block_table, int32_t max_blocks,
                                   const int32_t* seqlens, int32_t batch, int32_t q_len,
                                   int64_t max_seqlen, float softmax_scale, int32_t num_splits,
                                   void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                   void* out, void* stream) {
  return xmla_decode_profiled(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens,
                              batch, q_len, max_seqlen, softmax_scale, num_splits, workspace,
                              workspace_bytes, status_dev, out, stream, nullptr, nullptr);
}

// ---------------------------------------------------------------- decode without caller scratch

namespace xmla {

// Fixed device scratch for xmla_decode_noalloc.  It is part of the library's
// module image, so every GPU that loads the library holds it until the
// process exits; its size is the largest workspace that entry point accepts.
constexpr size_t kNoAllocScratchBytes = (size_t)XMLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mutex;
static void* g_noalloc_addr[64] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the real address is asked
// from the runtime once per device (with that device current) and cached.
static xmla_status noalloc_scratch(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return XMLA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return XMLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return XMLA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return XMLA_OK;
}

}  // namespace xmla

extern "C" xmla_status xmla_decode_noalloc(const xmla_yarn_cfg* cfg, const void* q,
                                           const void* W_UK, const void* W_UV, const void* pool,
                                           int64_t num_blocks, const int32_t* block_table,
                                           int32_t max_blocks, const int32_t* seqlens,
                                           int32_t batch, int32_t q_len, int64_t max_seqlen,
                                           float softmax_scale, int32_t num_splits,
                                           int32_t* status_dev, void* out, void* stream) {
  int nsm = 0;
  if (!xmla::device_ok(&nsm)) return XMLA_ERR_UNSUPPORTED;
  const size_t need = xmla_decode_workspace_size(batch, q_len, max_seqlen, nsm, num_splits);
  if (need == 0) return XMLA_ERR_SHAPE;
  if (need > xmla::kNoAllocScratchBytes) return XMLA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const xmla_status st = xmla::noalloc_scratch(&scratch);
  if (st != XMLA_OK) return st;
  return xmla_decode(cfg, q, W_UK, W_UV, pool, num_blocks, block_table, max_blocks, seqlens, batch,
                     q_len, max_seqlen, softmax_scale, num_splits, scratch,
                     xmla::kNoAllocScratchBytes, status_dev, out, stream);
}

extern "C" xmla_status xmla_selftest_wait_timeout(int32_t* status_dev, uint64_t timeout_ns,
                                                  void* stream) {
  if (status_dev == nullptr) return XMLA_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(status_dev, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
}

extern "C" const char* xmla_status_string(xmla_status s) {
  switch (s) {
    case XMLA_OK: return "ok";
    case XMLA_ERR_INVALID_ARG: return "invalid argument";
    case XMLA_ERR_SHAPE: return "unsupported shape";
    case XMLA_ERR_WORKSPACE: return "workspace too small";
    case XMLA_ERR_CUDA: return "CUDA error";
    case XMLA_ERR_DEVICE_OOB: return "device: index out of range";
    case XMLA_ERR_TIMEOUT: return "device: bounded wait timed out";
    case XMLA_ERR_UNSUPPORTED: return "device not supported (needs sm_100a)";
  }
  return "unknown status";
}
