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
// Three kernels per call:
//   q_absorb   q_ext[b,j,h] = c * [W_UK[h]^T q_nope | rope(q_pe)]   (c = scale * log2 e)
//   decode     one CTA per (sequence, row group, KV split): 64-token pages are
//              streamed by TMA into shared memory; S^T = page . q_ext^T (M = 64
//              tokens, N = rows, K = 576) and O^T += c_kv^T . P^T (M = 128 latent
//              dims x 4, N = rows, K = 64 tokens) run on tcgen05 with fp32
//              accumulators in tensor memory; the online softmax (base 2, lazy
//              max update) runs in registers.  Writes per-split (m, l, O).
//   combine    merges the splits by their log-sum-exp and applies W_UV[h].
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "xmla_device.cuh"
#include "yarn.cuh"

namespace xmla {

constexpr float kLog2e = 1.4426950408889634f;
// A row's running maximum is only raised when a score exceeds it by more than
// this (log2 units), so probabilities stay <= 2^kLazyMax before normalisation.
constexpr float kLazyMax = 8.0f;
constexpr int kMaxSplits = 1024;
constexpr int kSoftmaxThreads = 128;
constexpr int kDecodeThreads = 64 + kSoftmaxThreads;

// ---------------------------------------------------------------- shared-memory plan

template <int NR>
struct DecodeLayout {
  static_assert(NR == 32 || NR == 64, "rows per CTA");
  static constexpr int kLatSlots = NR == 32 ? 9 : 7;   // 16 KB: latent dims 128m..128m+127 of a page
  static constexpr int kRopeSlots = NR == 32 ? 4 : 2;  // 8 KB: rope dims of a page
  static constexpr uint32_t kQChunk = NR * 128;        // one 64-column chunk of q_ext
  static constexpr uint32_t kPBytes = NR * 128;        // P^T: NR rows x 64 tokens bf16
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
  static constexpr int kBarSFull = kBarRopeEmpty + kRopeSlots;
  static constexpr int kBarSFree = kBarSFull + 1;
  static constexpr int kBarPFull = kBarSFree + 1;   // 2
  static constexpr int kBarPvDone = kBarPFull + 2;  // 2
  static constexpr int kBarDrain = kBarPvDone + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr uint32_t kOffMUsed = (kOffBars + kNumBars * 8 + 15) & ~15u;
  static constexpr uint32_t kOffMNext = kOffMUsed + NR * 4;
  static constexpr uint32_t kOffAlpha = kOffMNext + NR * 4;
  static constexpr uint32_t kOffRed = kOffAlpha + NR * 4;
  static constexpr uint32_t kOffTmem = kOffRed + 4 * NR * 4;
  static constexpr uint32_t kOffAbort = kOffTmem + 4;
  static constexpr uint32_t kBytes = kOffAbort + 12;
  static constexpr uint32_t kSmem = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kSmem <= 232448, "shared memory per CTA");
  // tensor memory columns: O^T at [0, 4 NR), S^T at [4 NR, 5 NR)
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = 4 * NR;
  static constexpr uint32_t kTmemCols = 5 * NR <= 256 ? 256 : 512;
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

  // ---- setup
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
    mbar_init(bar(L::kBarSFull), 1);
    mbar_init(bar(L::kBarSFree), kSoftmaxThreads);
    mbar_init(bar(L::kBarPFull + 0), kSoftmaxThreads);
    mbar_init(bar(L::kBarPFull + 1), kSoftmaxThreads);
    mbar_init(bar(L::kBarPvDone + 0), 1);
    mbar_init(bar(L::kBarPvDone + 1), 1);
    mbar_init(bar(L::kBarDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + NR) m_used[threadIdx.x - 64] = -INFINITY;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  const int32_t qrow0 = (int32_t)(((int64_t)b * p.q_len + j0) * 32);

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0 && n_pages > 0) {
      tma_prefetch_desc(&tmap_pool);
      tma_prefetch_desc(&tmap_q);
      const uint64_t stream_policy = policy_evict_first();
      mbar_arrive_expect_tx(bar(L::kBarQ), 9u * L::kQChunk);
      for (int c = 0; c < 9; ++c)
        tma_load_2d(base + L::kOffQ + c * L::kQChunk, &tmap_q, c * 64, qrow0, bar(L::kBarQ));
      int li = 0, ri = 0;
      uint32_t lph = 0, rph = 0;
      int64_t lat_issued = 0, rope_issued = 0;
      bool ok = true;
      for (int i = 0; i < n_pages && ok; ++i) {
        int32_t blk = p.block_table[(int64_t)b * p.max_blocks + p_begin + i];
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
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0 && n_pages > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(64, NR, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, NR, true, false);
      const uint32_t t_s = tmem_base + L::kColS;
      const uint32_t t_o = tmem_base + L::kColO;
      bool ok = mbar_wait(bar(L::kBarQ), 0, abort_flag, p.status, p.wait_limit_ns);
      tc_fence_after();
      int li = 0, ri = 0;
      uint32_t lph = 0, rph = 0;
      for (int i = 0; i < n_pages && ok; ++i) {
        if (i > 0) {
          ok = mbar_wait(bar(L::kBarSFree), (uint32_t)((i - 1) & 1), abort_flag, p.status,
                         p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
        }
        // S^T[64 tok, NR] = page[64, 576] . q_ext[NR, 576]^T
        for (int m = 0; m < 4 && ok; ++m) {
          int s = li + m;
          uint32_t ph = lph;
          if (s >= L::kLatSlots) { s -= L::kLatSlots; ph ^= 1u; }
          ok = mbar_wait(bar(L::kBarLatFull + s), ph, abort_flag, p.status, p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t slot = base + L::kOffLat + s * L::kLatBytes;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int c = 2 * m + half;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t a = smem_desc_sw128(slot + half * 8192 + k * 32, 16, 1024);
              const uint64_t bq = smem_desc_sw128(base + L::kOffQ + c * L::kQChunk + k * 32, 16, 1024);
              tc_mma_bf16(t_s, a, bq, idesc_qk, (c | k) != 0 ? 1u : 0u);
            }
          }
        }
        if (!ok) break;
        ok = mbar_wait(bar(L::kBarRopeFull + ri), rph, abort_flag, p.status, p.wait_limit_ns);
        if (!ok) break;
        tc_fence_after();
        {
          const uint32_t slot = base + L::kOffRope + ri * L::kRopeBytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t a = smem_desc_sw128(slot + k * 32, 16, 1024);
            const uint64_t bq = smem_desc_sw128(base + L::kOffQ + 8 * L::kQChunk + k * 32, 16, 1024);
            tc_mma_bf16(t_s, a, bq, idesc_qk, 1u);
          }
        }
        tc_commit(bar(L::kBarSFull));
        tc_commit(bar(L::kBarRopeEmpty + ri));
        if (++ri == L::kRopeSlots) { ri = 0; rph ^= 1u; }

        // O^T[512, NR] += c_kv^T[512, 64 tok] . P^T[64 tok, NR]
        ok = mbar_wait(bar(L::kBarPFull + (i & 1)), (uint32_t)((i >> 1) & 1), abort_flag, p.status,
                       p.wait_limit_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t pbuf = base + L::kOffP + (i & 1) * L::kPBytes;
        for (int m = 0; m < 4; ++m) {
          int s = li + m;
          if (s >= L::kLatSlots) s -= L::kLatSlots;
          const uint32_t slot = base + L::kOffLat + s * L::kLatBytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t a = smem_desc_sw128(slot + k * 2048, 8192, 1024);
            const uint64_t bp = smem_desc_sw128(pbuf + k * 32, 16, 1024);
            tc_mma_bf16(t_o + m * NR, a, bp, idesc_pv, (i > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(bar(L::kBarLatEmpty + s));
        }
        tc_commit(bar(L::kBarPvDone + (i & 1)));
        li += 4;
        if (li >= L::kLatSlots) { li -= L::kLatSlots; lph ^= 1u; }
      }
      // all issued tensor-core work must finish before tensor memory is freed
      tc_commit(bar(L::kBarDrain));
      mbar_wait(bar(L::kBarDrain), 0, nullptr, p.status, p.wait_limit_ns);
    }
  } else {
    // ================================================================ softmax / epilogue
    const int tid = threadIdx.x - 64;
    const int quarter = warp & 3;            // tensor-memory lane quarter this warp may access
    const int tok = 16 * quarter + lane;     // token of the page held by this thread (lane < 16)
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quarter) << 16);
    float l_part[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) l_part[n] = 0.f;
    const int64_t qpos0 = seqlen - p.q_len + j0;  // position of this CTA's first query
    bool ok = true;
    for (int i = 0; i < n_pages; ++i) {
      ok = mbar_wait(bar(L::kBarSFull), (uint32_t)(i & 1), abort_flag, p.status, p.wait_limit_ns);
      if (named_bar_or(1, kSoftmaxThreads, !ok)) { ok = false; break; }
      tc_fence_after();
      float sv[NR];
#pragma unroll
      for (int c = 0; c < NR / 32; ++c) {
        float tmp[32];
        tmem_ld32(t_lane + L::kColS + 32 * c, tmp);
#pragma unroll
        for (int k = 0; k < 32; ++k) sv[32 * c + k] = tmp[k];
      }
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::kBarSFree));

      const int64_t tpos = (p_begin + i) * kPage + tok;
      bool exceed = false;
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const bool vis = lane < 16 && (n >> 5) < jn && tpos <= qpos0 + (n >> 5);
        sv[n] = vis ? sv[n] : -INFINITY;
        exceed |= sv[n] > m_used[n] + kLazyMax;
      }
      if (named_bar_or(1, kSoftmaxThreads, exceed)) {
#pragma unroll
        for (int c = 0; c < NR / 32; ++c) {
          float tmp[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) tmp[k] = sv[32 * c + k];
          xpose_reduce32<true>(tmp, lane);
          red[quarter * NR + 32 * c + lane] = tmp[0];
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
        for (int n = 0; n < NR; ++n) l_part[n] *= alpha_s[n];
        if (tid < NR) m_used[tid] = m_next[tid];
        named_bar_sync(1, kSoftmaxThreads);
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
      uint8_t* pbuf = smem + L::kOffP + (i & 1) * L::kPBytes;
#pragma unroll
      for (int n = 0; n < NR; ++n) {
        const float pr = sv[n] == -INFINITY ? 0.f : ex2(sv[n] - m_used[n]);
        const __nv_bfloat16 hb = __float2bfloat16_rn(pr);
        l_part[n] += __bfloat162float(hb);
        if (lane < 16) *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128_offset(n, tok)) = hb;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::kBarPFull + (i & 1)));
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
        float tmp[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) tmp[k] = l_part[32 * c + k];
        xpose_reduce32<false>(tmp, lane);
        red[quarter * NR + 32 * c + lane] = tmp[0];
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
// entries).  grid (32 heads, 4 column blocks of 128); block 128 threads, one
// latent column each; the column-block-0 CTAs also rotate the rope part.
constexpr int kAbsorbRows = 32;

__global__ void __launch_bounds__(128) q_absorb_kernel(const __nv_bfloat16* __restrict__ q,
                                                       const __nv_bfloat16* __restrict__ W_UK,
                                                       const int32_t* __restrict__ seqlens,
                                                       __nv_bfloat16* __restrict__ q_ext, int rows,
                                                       int q_len, float qscale,
                                                       const RopeTable tab) {
  __shared__ float sq[kAbsorbRows][kDNope];
  const int h = blockIdx.x;
  const int col = blockIdx.y * 128 + threadIdx.x;
  float w[kDNope];
#pragma unroll
  for (int d = 0; d < kDNope; ++d)
    w[d] = __bfloat162float(W_UK[((int64_t)h * kDNope + d) * kDLatent + col]);
  for (int r0 = 0; r0 < rows; r0 += kAbsorbRows) {
    const int nr = min(kAbsorbRows, rows - r0);
    __syncthreads();
    for (int e = threadIdx.x; e < nr * kDNope; e += blockDim.x) {
      const int r = e / kDNope, d = e % kDNope;
      sq[r][d] = __bfloat162float(q[((int64_t)(r0 + r) * kHeads + h) * kDQ + d]);
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < kDNope; ++d) acc = fmaf(sq[r][d], w[d], acc);
      q_ext[((int64_t)(r0 + r) * kHeads + h) * kDRow + col] = __float2bfloat16_rn(acc * qscale);
    }
  }
  if (blockIdx.y == 0) {
    constexpr int kPairs = kDRope / 2;
    for (int e = threadIdx.x; e < rows * kPairs; e += blockDim.x) {
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
  }
}

// ---------------------------------------------------------------- combine + W_UV

// One CTA (128 threads) per output row (b, j, h): merge the splits' partial
// latent outputs by their log-sum-exp, then out = o_lat . W_UV[h].
__global__ void __launch_bounds__(128) combine_uv_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_ml,
                                                         const __nv_bfloat16* __restrict__ W_UV,
                                                         __nv_bfloat16* __restrict__ out, int q_len,
                                                         int groups, int nsplit, int rows_per_cta) {
  __shared__ float w_s[kMaxSplits];
  __shared__ float o_lat[kDLatent];
  __shared__ float red_s[4];
  const int row = blockIdx.x;  // (b*q_len + j)*32 + h
  const int h = row % kHeads;
  const int bj = row / kHeads;
  const int j = bj % q_len;
  const int b = bj / q_len;
  const int r = j * kHeads + h;
  const int g = r / rows_per_cta;
  const int n = r % rows_per_cta;
  const int64_t item0 = ((int64_t)b * groups + g) * nsplit;
  const int tid = threadIdx.x;

  // global max over splits that saw any token
  float mx = -INFINITY;
  for (int s = tid; s < nsplit; s += blockDim.x) {
    const float m = part_ml[((item0 + s) * rows_per_cta + n) * 2 + 0];
    const float l = part_ml[((item0 + s) * rows_per_cta + n) * 2 + 1];
    if (l > 0.f) mx = fmaxf(mx, m);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red_s[tid >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red_s[0], red_s[1]), fmaxf(red_s[2], red_s[3]));
  __syncthreads();
  float lsum = 0.f;
  for (int s = tid; s < nsplit; s += blockDim.x) {
    const float m = part_ml[((item0 + s) * rows_per_cta + n) * 2 + 0];
    const float l = part_ml[((item0 + s) * rows_per_cta + n) * 2 + 1];
    const float wgt = l > 0.f ? ex2(m - mx) : 0.f;
    w_s[s] = wgt;
    lsum += wgt * l;
  }
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if ((tid & 31) == 0) red_s[tid >> 5] = lsum;
  __syncthreads();
  lsum = red_s[0] + red_s[1] + red_s[2] + red_s[3];
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;

  // o_lat: thread handles 4 consecutive latent dims
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < nsplit; ++s) {
    const float wgt = w_s[s];
    if (wgt == 0.f) continue;
    const float4 v = reinterpret_cast<const float4*>(
        part_o + ((item0 + s) * rows_per_cta + n) * kDLatent)[tid];
    acc.x = fmaf(wgt, v.x, acc.x);
    acc.y = fmaf(wgt, v.y, acc.y);
    acc.z = fmaf(wgt, v.z, acc.z);
    acc.w = fmaf(wgt, v.w, acc.w);
  }
  o_lat[4 * tid + 0] = acc.x * inv;
  o_lat[4 * tid + 1] = acc.y * inv;
  o_lat[4 * tid + 2] = acc.z * inv;
  o_lat[4 * tid + 3] = acc.w * inv;
  __syncthreads();

  // out[v] = sum_c o_lat[c] W_UV[h][c][v], thread v
  const __nv_bfloat16* wv = W_UV + (int64_t)h * kDLatent * kDV + tid;
  float y = 0.f;
#pragma unroll 8
  for (int c = 0; c < kDLatent; ++c) y = fmaf(o_lat[c], __bfloat162float(wv[(int64_t)c * kDV]), y);
  out[(int64_t)row * kDV + tid] = __float2bfloat16_rn(y);
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
  mla_decode_kernel<NR><<<(unsigned)items, kDecodeThreads, L::kSmem, st>>>(tp, tq, dp);
  return cudaGetLastError();
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
  q_absorb_kernel<<<dim3(kHeads, kDLatent / 128), 128, 0, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)W_UK, seqlens, q_ext, rows, q_len, qscale,
      make_rope_table(cfg));
  if (cudaGetLastError() != cudaSuccess) return XMLA_ERR_CUDA;

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

  combine_uv_kernel<<<rows * kHeads, 128, 0, st>>>(dp.part_o, dp.part_ml,
                                                    (const __nv_bfloat16*)W_UV,
                                                    (__nv_bfloat16*)out, q_len, P.groups,
                                                    P.nsplit, P.nr);
  return cudaGetLastError() == cudaSuccess ? XMLA_OK : XMLA_ERR_CUDA;
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
