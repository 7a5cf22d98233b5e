// Split-K MLA decode attention over the 8-bit paged latent cache.
//
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 三,
//      方案 A: an 8-bit (q8_0) KV cache halves the bytes a long context costs.
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": the cache row is the 512-dim latent and the 64-dim rope key;
//      the absorbed form reads it once per step as [c_kv | k_pe].
//
// A cache row is 576 int8 codes and 18 block exponents (q8_append.cu): value =
// code * 2^e, exact in f16.  The same split-K scheme as the bf16 kernel
// (mla_decode.cu), with the page tiles made on chip:
//   * eight converter warps load each page's codes straight from global memory
//     (one warp covers 8 tokens x 64 columns per step: 16 fully used sectors
//     per load) and write it as f16 into a page buffer laid out exactly as the
//     128-byte-swizzled TMA tiles of the bf16 kernel (conflict-free: the 8
//     lanes of a store phase hold 8 rows of one swizzle atom);
//   * one converter lane keeps the next pages streaming into L2 with bulk
//     prefetches, so the converters' loads hit L2;
//   * two page buffers of 72 KB: the page after next is converted while the
//     tensor cores and the softmax work on the current one;
//   * QK and PV are f16 tcgen05 products (f32 accumulators in tensor memory),
//     q_ext is f16 (11 significant bits) and P is rounded to f16.
// Rows per CTA: 32 (one query's 32 heads).  Writes the split's (m, l, O) in
// the bf16 kernel's layout, so the combine is shared.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "decode_chain.h"
#include "split_kv.h"
#include "xmla_device.cuh"

namespace xmla {

namespace {

constexpr float kQ8LazyMax = 8.0f;  // as the bf16 kernel: a row max moves only by > 2^8
constexpr int kQ8SoftmaxThreads = 128;
constexpr int kQ8SoftmaxWarp0 = 3;  // warps: 0 q loader, 1 QK, 2 PV, 3-6 softmax, 7-14 convert
constexpr int kQ8ConvWarp0 = 7;
constexpr int kQ8ConvWarps = 8;
constexpr int kQ8Threads = 32 * (kQ8ConvWarp0 + kQ8ConvWarps);  // 480
constexpr int kQ8Ahead = 3;  // pages kept in flight into L2 ahead of the converters
constexpr uint32_t kQ8PageBytes = kPage * kQ8Row;  // 38912

struct Q8Layout {
  static constexpr int NR = 32;
  static constexpr uint32_t kQChunk = NR * 128;         // 64 f16 columns of q_ext, 32 rows
  static constexpr uint32_t kPRow = NR * 2;             // P^T row: 32 f16 (64-byte swizzle)
  static constexpr uint32_t kPBytes = 64 * kPRow;
  static constexpr uint32_t kPGroup = 8 * kPRow;
  static constexpr uint32_t kChunk = 8192;              // 64 tokens x 64 f16 columns
  static constexpr uint32_t kPageBuf = 9 * kChunk;      // latent chunks 0..7, rope chunk 8
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffP = kOffQ + 9 * kQChunk;
  static constexpr uint32_t kOffPage = kOffP + 2 * kPBytes;
  static constexpr uint32_t kOffBars = kOffPage + 2 * kPageBuf;
  static constexpr int kBarQ = 0;
  static constexpr int kBarFull = 1;     // 2: page buffer converted
  static constexpr int kBarSFull = 3;    // 2
  static constexpr int kBarSFree = 5;    // 2
  static constexpr int kBarPFull = 7;    // 2
  static constexpr int kBarPvDone = 9;   // 2
  static constexpr int kBarDrain = 11;   // 2: QK issuer, PV issuer
  static constexpr int kNumBars = 13;
  static constexpr uint32_t kOffMUsed = (kOffBars + kNumBars * 8 + 15) & ~15u;
  static constexpr uint32_t kOffMNext = kOffMUsed + NR * 4;
  static constexpr uint32_t kOffAlpha = kOffMNext + NR * 4;
  static constexpr uint32_t kOffRed = kOffAlpha + NR * 4;
  static constexpr uint32_t kOffTmem = kOffRed + 4 * NR * 4;
  static constexpr uint32_t kOffAbort = kOffTmem + 4;
  static constexpr uint32_t kBytes = kOffAbort + 12;
  static constexpr uint32_t kSmem = kBytes + 1024;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(kOffP % 1024 == 0 && kOffPage % 1024 == 0, "alignment");
  static constexpr uint32_t kColO = 0;       // O^T: 4 tiles of M=128 x N=32
  static constexpr uint32_t kColS = 4 * NR;  // two S^T buffers of 32 columns
  static constexpr uint32_t kTmemCols = 256;
};

// Over the 16 threads of one row parity (lane bits 0, 2, 3, 4): on return v[0]
// holds the reduction of value j = b0 + 2 b2 + 4 b3 + 8 b4.  (The bf16 kernel's
// copy stays in its own translation unit: that kernel's code generation has
// proven sensitive to changes around it.)
template <bool kMax>
__device__ __forceinline__ void q8_xpose_reduce16(float (&v)[16], int lane) {
  constexpr int kMask[4] = {16, 8, 4, 1};
#pragma unroll
  for (int lv = 0; lv < 4; ++lv) {
    const int w = 8 >> lv;
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

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Four int8 codes -> two f16x2 words of code * 2^e.  (code + 128) placed under
// the f16 exponent of 1024 reads as 1152 + code; subtracting 1152 and scaling
// by the power of two 2^e (|code| <= 128, e in [-14, 8]) are both exact.
__device__ __forceinline__ void q8_to_f16x4(uint32_t w, __half2 scale, uint32_t& lo,
                                            uint32_t& hi) {
  const uint32_t x = w ^ 0x80808080u;
  const uint32_t a = __byte_perm(x, 0x64646464u, 0x4140);
  const uint32_t b = __byte_perm(x, 0x64646464u, 0x4342);
  const __half2 bias = __half2half2(__ushort_as_half((unsigned short)0x6480));  // 1152
  const __half2 ra = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&a), bias), scale);
  const __half2 rb = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&b), bias), scale);
  lo = *reinterpret_cast<const uint32_t*>(&ra);
  hi = *reinterpret_cast<const uint32_t*>(&rb);
}

}  // namespace

template <int kMode>
__global__ void __launch_bounds__(kQ8Threads, 1)
    mla_decode_q8_kernel(const __grid_constant__ CUtensorMap tmap_q, const DecodeParams p,
                         const uint8_t* __restrict__ pool_q8) {
  using L = Q8Layout;
  constexpr int NR = L::NR;
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

  // ---- work item: (sequence b, query g, split) or a work-table entry
  const int item = blockIdx.x;
  int b = 0, g = 0;
  int64_t seqlen = 0, npages = 0, p_begin = 0, p_end = 0;
  if constexpr (kMode == 0) {
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
    const int64_t pps = (npages + p.nsplit - 1) / p.nsplit;
    p_begin = (int64_t)split * pps;
    p_end = min(npages, p_begin + pps);
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQ), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::kBarFull + i), kQ8ConvWarps);
      mbar_init(bar(L::kBarSFull + i), 1);
      mbar_init(bar(L::kBarSFree + i), kQ8SoftmaxThreads);
      mbar_init(bar(L::kBarPFull + i), kQ8SoftmaxThreads);
      mbar_init(bar(L::kBarPvDone + i), 1);
      mbar_init(bar(L::kBarDrain + i), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::kOffTmem, L::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 32 * kQ8SoftmaxWarp0 && threadIdx.x < 32 * kQ8SoftmaxWarp0 + NR)
    m_used[threadIdx.x - 32 * kQ8SoftmaxWarp0] = -INFINITY;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  if constexpr (kMode != 0) {
    // the table comes from the kernel launched before this one
    pdl_wait();
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
  const int j0 = g;  // one query per CTA
  // causal: pages past this query's position hold nothing it may see
  p_end = min(p_end, (seqlen - p.q_len + j0) / kPage + 1);
  const int n_pages = (int)max((int64_t)0, p_end - p_begin);
  const int32_t qrow0 = (int32_t)(((int64_t)b * p.q_len + j0) * kHeads);
  const int32_t* bt = p.block_table + (int64_t)b * p.max_blocks + p_begin;
  pdl_launch_dependents();

  if (warp == 0) {
    // ================================================================ q_ext loader
    if (lane == 0 && n_pages > 0) {
      tma_prefetch_desc(&tmap_q);
      pdl_wait();  // q_ext comes from the kernel launched before this one
      mbar_arrive_expect_tx(bar(L::kBarQ), 9u * L::kQChunk);
      for (int c = 0; c < 9; ++c)
        tma_load_2d(base + L::kOffQ + c * L::kQChunk, &tmap_q, c * 64, qrow0, bar(L::kBarQ));
      mbar_wait(bar(L::kBarQ), 0, nullptr, p.status, p.wait_limit_ns);
    }
  } else if (warp >= kQ8ConvWarp0) {
    // ================================================================ converters
    const int cw = warp - kQ8ConvWarp0;
    const int tok = 8 * cw + (lane & 7);  // token of the page this lane converts
    const int jq = lane >> 3;             // 16-code vector within a 64-column chunk
    const int sw = tok & 7;               // 128-byte swizzle phase of the token's rows
    auto page_ptr = [&](int i, bool& valid) -> const uint8_t* {
      const int32_t blk = bt[i];
      valid = blk >= 0 && (int64_t)blk < p.num_blocks;
      return pool_q8 + (int64_t)(valid ? blk : 0) * kQ8PageBytes;
    };
    if (cw == 0 && lane == 0) {
      // the cache pages are final once the kernels before this one are done;
      // an L2 prefetch before that point only warms lines a later write updates
      for (int a = 0; a < kQ8Ahead && a < n_pages; ++a) {
        bool v;
        const uint8_t* pg = page_ptr(a, v);
        if (v) prefetch_l2_bulk(pg, kQ8PageBytes);
      }
    }
    pdl_wait();
    bool ok = true;
    for (int i = 0; i < n_pages && ok; ++i) {
      bool valid;
      const uint8_t* pg = page_ptr(i, valid);
      if (!valid && cw == 0 && lane == 0) record_status(p.status, XMLA_ERR_DEVICE_OOB);
      const uint8_t* row = pg + tok * kQ8Row;
      uint4 v[9];
      uint4 ex0 = make_uint4(0u, 0u, 0u, 0u);
      uint2 ex1 = make_uint2(0u, 0u);
      if (valid) {
#pragma unroll
        for (int c = 0; c < 9; ++c) v[c] = ld_stream_v4(row + c * 64 + jq * 16);
        ex0 = ld_stream_v4(row + kDRow);        // exponents of blocks 0..15
        ex1 = ld_stream_v2(row + kDRow + 16);   // blocks 16, 17 (and pad)
      } else {
#pragma unroll
        for (int c = 0; c < 9; ++c) v[c] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (cw == 0 && lane == 0 && i + kQ8Ahead < n_pages) {
        bool va;
        const uint8_t* pa = page_ptr(i + kQ8Ahead, va);
        if (va) prefetch_l2_bulk(pa, kQ8PageBytes);
      }
      // page buffer i & 1 is free once the PV of page i - 2 has completed
      if (i >= 2) {
        bool okw = true;
        if (lane == 0) {
          const int pi = i - 2;
          okw = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1), abort_flag,
                          p.status, p.wait_limit_ns);
        }
        ok = __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      uint8_t* buf = smem + L::kOffPage + (i & 1) * L::kPageBuf + tok * 128;
      // the exponent of block 2c + (jq >> 1) is byte 2(c & 1) + (jq >> 1) of word c >> 1
      const int ex_shift = 8 * (jq >> 1);
#pragma unroll
      for (int c = 0; c < 9; ++c) {
        const uint32_t ew = c < 2 ? ex0.x : c < 4 ? ex0.y : c < 6 ? ex0.z : c < 8 ? ex0.w : ex1.x;
        int e = (int)(int8_t)((ew >> (16 * (c & 1) + ex_shift)) & 0xffu);
        e = min(max(e, kQ8EMin), kQ8EMax);
        uint32_t o[8];
        if (e <= 5) {
          // (code + 128) under the f16 exponent 25 + e reads 2^(e+10) + (code+128) 2^e;
          // subtracting 1152 * 2^e (exact: both lie in [2^(e+10), 2^(e+11))) leaves
          // code * 2^e, one operation fewer per pair than the general path
          const uint32_t magic = (uint32_t)((25 + e) << 2) * 0x01010101u;
          const __half2 sub =
              __half2half2(__ushort_as_half((unsigned short)(((25 + e) << 10) | 0x80)));
          const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t x = wv[q] ^ 0x80808080u;
            const uint32_t a = __byte_perm(x, magic, 0x4140), bb = __byte_perm(x, magic, 0x4342);
            const __half2 ra = __hsub2(*reinterpret_cast<const __half2*>(&a), sub);
            const __half2 rb = __hsub2(*reinterpret_cast<const __half2*>(&bb), sub);
            o[2 * q] = *reinterpret_cast<const uint32_t*>(&ra);
            o[2 * q + 1] = *reinterpret_cast<const uint32_t*>(&rb);
          }
        } else {
          const __half2 scale = __half2half2(__ushort_as_half((unsigned short)((e + 15) << 10)));
          q8_to_f16x4(v[c].x, scale, o[0], o[1]);
          q8_to_f16x4(v[c].y, scale, o[2], o[3]);
          q8_to_f16x4(v[c].z, scale, o[4], o[5]);
          q8_to_f16x4(v[c].w, scale, o[6], o[7]);
        }
        uint8_t* dst = buf + c * L::kChunk;
        *reinterpret_cast<uint4*>(dst + (((2 * jq) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(dst + (((2 * jq + 1) ^ sw) << 4)) =
            make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarFull + (i & 1)));
    }
  } else if (warp == 1 || warp == 2) {
    // ================================================================ tensor-core issuers
    if (lane == 0 && n_pages > 0) {
      // tc_mma_bf16 issues tcgen05.mma kind::f16; the operand type (f16 here) is
      // the instruction descriptor's
      constexpr uint32_t idesc_qk = idesc_f16_f32(64, NR, false, false);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, NR, true, true);
      const uint64_t d_page_k = smem_desc_sw128(base + L::kOffPage, 16, 1024);     // K-major
      const uint64_t d_page_mn = smem_desc_sw128(base + L::kOffPage, 8192, 1024);  // c_kv^T
      const uint64_t d_q = smem_desc_sw128(base + L::kOffQ, 16, 1024);
      const uint64_t d_p = smem_desc(base + L::kOffP, 8192, L::kPGroup, kSwizzle64B);
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
          }
          if (!(ok = wait(L::kBarFull + sb, (uint32_t)((i >> 1) & 1)))) break;
          tc_fence_after();
          const uint32_t t_s = tmem_base + L::kColS + sb * NR;
          const uint64_t a0 = d_page_k + ((sb * L::kPageBuf) >> 4);
#pragma unroll
          for (int c = 0; c < 9; ++c) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(t_s, a0 + ((c * L::kChunk + k * 32) >> 4),
                          d_q + ((c * L::kQChunk + k * 32) >> 4), idesc_qk, (c | k) != 0 ? 1u : 0u);
          }
          tc_commit(bar(L::kBarSFull + sb));
        }
      } else {
        for (int i = 0; i < n_pages && ok; ++i) {
          const int sb = i & 1;
          if (!(ok = wait(L::kBarPFull + sb, (uint32_t)((i >> 1) & 1)))) break;
          tc_fence_after();
          const uint64_t bp = d_p + ((sb * L::kPBytes) >> 4);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint64_t a0 = d_page_mn + ((sb * L::kPageBuf + m * 2 * L::kChunk) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(tmem_base + L::kColO + m * NR, a0 + ((k * 2048) >> 4),
                          bp + ((k * 2 * L::kPGroup) >> 4), idesc_pv, (i > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(bar(L::kBarPvDone + sb));
        }
      }
      const int drain = L::kBarDrain + (warp - 1);
      tc_commit(bar(drain));
      mbar_wait(bar(drain), 0, nullptr, p.status, p.wait_limit_ns);
    }
  } else {
    // ================================================================ softmax / epilogue
    // As the bf16 kernel: thread t of a softmax warp holds token
    // 8*(t&1) + (t>>2) of its tensor-memory quarter and the 16 rows of one
    // parity, n = pr + 2j.
    constexpr int kV = NR / 2;
    constexpr int kH = kV / 2;
    const int tid = threadIdx.x - 32 * kQ8SoftmaxWarp0;
    const int quarter = warp & 3;
    const int pr = (lane >> 1) & 1;
    const int tok = 16 * quarter + 8 * (lane & 1) + (lane >> 2);
    const int row_t = (lane & 1) + 2 * ((lane >> 2) & 1) + 4 * ((lane >> 3) & 1) + 8 * ((lane >> 4) & 1);
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quarter) << 16);
    float l_part[kV], mr[kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      l_part[j] = 0.f;
      mr[j] = -INFINITY;
    }
    const int64_t qpos = seqlen - p.q_len + j0;  // this CTA's query position
    bool ok = true;
    for (int i = 0; i < n_pages; ++i) {
      const int sb = i & 1;
      ok = mbar_wait(bar(L::kBarSFull + sb), (uint32_t)((i >> 1) & 1), abort_flag, p.status,
                     p.wait_limit_ns);
      tc_fence_after();
      float sv[kV];
      tmem_ld16x64b_x16(t_lane + L::kColS + sb * NR, sv);
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(L::kBarSFree + sb));

      bool exceed = false;
      if ((p_begin + i + 1) * kPage - 1 <= qpos) {
#pragma unroll
        for (int j = 0; j < kV; ++j) exceed |= sv[j] > mr[j] + kQ8LazyMax;
      } else {
        const bool vis = (p_begin + i) * kPage + tok <= qpos;
#pragma unroll
        for (int j = 0; j < kV; ++j) {
          sv[j] = vis ? sv[j] : -INFINITY;
          exceed |= sv[j] > mr[j] + kQ8LazyMax;
        }
      }
      bool okp = true;
      if (i >= 2) {
        const int pi = i - 2;
        okp = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1), abort_flag,
                        p.status, p.wait_limit_ns);
      }
      if (named_bar_or(1, kQ8SoftmaxThreads, exceed || !ok || !okp)) {
        if (named_bar_or(1, kQ8SoftmaxThreads, !ok || !okp)) { ok = false; break; }
        {
          float tmp[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) tmp[k] = sv[k];
          q8_xpose_reduce16<true>(tmp, lane);
          red[quarter * NR + pr + 2 * row_t] = tmp[0];
        }
        named_bar_sync(1, kQ8SoftmaxThreads);
        if (tid < NR) {
          const float mo = m_used[tid];
          float mn = mo;
#pragma unroll
          for (int q = 0; q < 4; ++q) mn = fmaxf(mn, red[q * NR + tid]);
          m_next[tid] = mn;
          alpha_s[tid] = (mn == -INFINITY) ? 1.f : ex2(mo - mn);
        }
        named_bar_sync(1, kQ8SoftmaxThreads);
        if (i > 0) {
          const int pi = i - 1;
          const bool okw = mbar_wait(bar(L::kBarPvDone + (pi & 1)), (uint32_t)((pi >> 1) & 1),
                                     abort_flag, p.status, p.wait_limit_ns);
          if (named_bar_or(1, kQ8SoftmaxThreads, !okw)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
            float o[32];
            const uint32_t ta = t_lane + L::kColO + m * NR;
            tmem_ld32(ta, o);
            tc_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] *= alpha_s[k];
            tmem_st32(ta, o);
          }
          tc_wait_st();
        }
#pragma unroll
        for (int j = 0; j < kV; ++j) l_part[j] *= alpha_s[pr + 2 * j];
        if (tid < NR) m_used[tid] = m_next[tid];
        named_bar_sync(1, kQ8SoftmaxThreads);
#pragma unroll
        for (int j = 0; j < kV; ++j) mr[j] = m_used[pr + 2 * j];
      }
      // probabilities rounded to f16 in pairs and summed in that precision
      uint32_t x[kH];
#pragma unroll
      for (int k = 0; k < kH; ++k) {
        const float p0 = sv[k] == -INFINITY ? 0.f : ex2(sv[k] - mr[k]);
        const float p1 = sv[kH + k] == -INFINITY ? 0.f : ex2(sv[kH + k] - mr[kH + k]);
        const __half2 hv = __floats2half2_rn(p0, p1);
        x[k] = *reinterpret_cast<const uint32_t*>(&hv);
        l_part[k] += __low2float(hv);
        l_part[kH + k] += __high2float(hv);
      }
      uint32_t w[kH];
#pragma unroll
      for (int k = 0; k < kH; ++k) {
        const uint32_t rcv = __shfl_xor_sync(0xffffffffu, x[k], 2);
        w[k] = pr == 0 ? __byte_perm(x[k], rcv, 0x5410) : __byte_perm(rcv, x[k], 0x7632);
      }
      uint8_t* prow = smem + L::kOffP + sb * L::kPBytes + tok * L::kPRow;
#pragma unroll
      for (int u = 0; u < kH / 4; ++u) {
        const int unit = pr * (kH / 4) + u;
        const int phys = unit ^ ((tok >> 1) & 3);
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
      have = !named_bar_or(1, kQ8SoftmaxThreads, !okw);
    }
    if (have) {
      tc_fence_after();
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + 32 * quarter + lane;
        float o[32];
        tmem_ld32(t_lane + L::kColO + m * NR, o);
        tc_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) p.part_o[(row0 + k) * kDLatent + d] = o[k];
      }
      {
        float tmp[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) tmp[k] = l_part[k];
        q8_xpose_reduce16<false>(tmp, lane);
        red[quarter * NR + pr + 2 * row_t] = tmp[0];
      }
      named_bar_sync(1, kQ8SoftmaxThreads);
      if (tid < NR) {
        const float l = red[tid] + red[NR + tid] + red[2 * NR + tid] + red[3 * NR + tid];
        p.part_ml[(row0 + tid) * 2 + 0] = m_used[tid];
        p.part_ml[(row0 + tid) * 2 + 1] = l;
      }
    } else if (tid < NR) {
      pdl_wait();  // the previous step's merge may still read this split's m, l
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

template <int kMode>
static cudaError_t launch_q8(const CUtensorMap& tq, const DecodeParams& dp, const uint8_t* pool_q8,
                             int64_t items, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(mla_decode_q8_kernel<kMode>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Q8Layout::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return launch_pdl(mla_decode_q8_kernel<kMode>, dim3((unsigned)items), dim3(kQ8Threads),
                    Q8Layout::kSmem, st, tq, dp, pool_q8);
}

cudaError_t launch_split_kv_q8(const CUtensorMap& q_map, const DecodeParams& dp,
                               const uint8_t* pool_q8, int64_t items, cudaStream_t st) {
  if (pool_q8 == nullptr) return cudaErrorInvalidValue;
  return dp.work_tab != nullptr ? launch_q8<1>(q_map, dp, pool_q8, items, st)
                                : launch_q8<0>(q_map, dp, pool_q8, items, st);
}

}  // namespace xmla
