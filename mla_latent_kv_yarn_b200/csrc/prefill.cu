// Prompt chunks in the non-absorbed form, on the tensor cores.
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": kv_b_proj expands K_nope and V per head (32 x (128 + 128)) from
//      the cached 512-dim latent; attention then runs per head over
//      [K_nope | rotated k_pe] (192 dims) and V (128 dims).
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 三 (方案 D):
//      prompt processing is what grows with the context.
//
// A decode step has one query per sequence and is bound by reading the cache
// once, which the absorbed form does.  A prompt chunk has hundreds or
// thousands of queries per sequence, and every cached token is attended by all
// of them: the work is the products, and the non-absorbed form needs 2 x (192
// + 128) flop per (query, token, head) against 2 x (576 + 512) absorbed.  A
// chunk runs three kernels, chained with programmatic dependent launch:
//   prep    the queries as fp16 rows [q_nope | rope(q_pe)] (and, for a decode
//           step, the append of the chunk's cache rows);
//   expand  K_nope[t, h] = W_UK[h] c_kv[t] and V[t, h] = W_UV[h]^T c_kv[t] for
//           every cached token of each sequence, a tcgen05 GEMM (bf16 inputs,
//           fp32 accumulators) written as fp16, and the rotated rope key
//           copied out as fp16;
//   attend  per (sequence, head, tile of 128 queries): flash-style attention
//           over tiles of 128 tokens, S = Q K^T and O += P V on tcgen05 with
//           fp16 operands and fp32 accumulators in tensor memory, one softmax
//           thread per query row, the output written directly (V already
//           carries W_UV).
// fp16 operands carry 11 significant bits: emulating these roundings on the
// CPU keeps every element of a fresh prompt within 1e-2 + 2^-8 |ref| of the
// fp64 definition, where bf16 operands (8 bits) do not.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>

#include "append.cuh"
#include "decode_chain.h"
#include "prefill.h"

namespace xmla {

namespace {

constexpr uint32_t kTile = 16384;  // one 128-row x 64-element box of 2-byte values (128-byte rows)

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int32_t x, int32_t y,
                                            int32_t z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// kind::f16 products take fp16 or bf16 operands; the instruction descriptor
// carries which (idesc_f16_f32 / idesc_bf16_f32)
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  tc_mma_bf16(d_tmem, a_desc, b_desc, idesc, accumulate);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ---------------------------------------------------------------- prep

constexpr int kPrepThreads = 256;
constexpr int kPrepRows = 2;  // query rows (all 32 heads) per block

// Blocks [0, ceil(rows / kPrepRows)): qh[r, h] = [q_nope | rope(q_pe, pos_r)]
// as fp16, pos_r = seqlens[b] - q_len + j for r = b * q_len + j (the angle in
// float64 once per (row, pair), as rope_pair).  The blocks after them append
// the chunk's ready cache rows (one thread per 16-byte piece, the rope key
// rotated on the way), as the decode step's first kernel does.
__global__ void __launch_bounds__(kPrepThreads)
    prefill_prep_kernel(const __nv_bfloat16* q, const int32_t* seqlens, __half* __restrict__ qh,
                        int rows, int q_len, const RopeTable q_tab, const AppendArgs ap,
                        const RopeTable k_tab) {
  __shared__ double cs[kPrepRows][kDRope / 2][2];
  pdl_wait();  // q, the lengths and the cache may come from the kernel launched before
  pdl_launch_dependents();
  const int t = threadIdx.x;
  const int q_blocks = (rows + kPrepRows - 1) / kPrepRows;
  if ((int)blockIdx.x < q_blocks) {
    const int r_lo = blockIdx.x * kPrepRows;
    const int nr = min(kPrepRows, rows - r_lo);
    constexpr int kPairs = kDRope / 2;
    if (t < nr * kPairs) {
      const int rr = t / kPairs, i = t % kPairs;
      const int r = r_lo + rr;
      const int64_t pos = (int64_t)seqlens[r / q_len] - q_len + (r % q_len);
      double s, c;
      sincos((double)pos * q_tab.inv_freq[i], &s, &c);
      cs[rr][i][0] = c * q_tab.magnitude;
      cs[rr][i][1] = s * q_tab.magnitude;
    }
    // q_nope: 16 pieces of 8 values per (row, head), converted while the
    // angles are formed
    for (int e = t; e < nr * kHeads * 16; e += kPrepThreads) {
      const int64_t rh = (int64_t)r_lo * kHeads + e / 16;
      const int u = e % 16;
      const uint4 v = *reinterpret_cast<const uint4*>(q + rh * kDQ + 8 * u);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int k = 0; k < 4; ++k) ow[k] = pack_half2(__low2float(b2[k]), __high2float(b2[k]));
      *reinterpret_cast<uint4*>(qh + rh * kDQ + 8 * u) = o;
    }
    __syncthreads();
    // rotated q_pe: pairs (i, i + 32) for four consecutive i per thread
    for (int e = t; e < nr * kHeads * (kPairs / 4); e += kPrepThreads) {
      const int rr = e / (kHeads * (kPairs / 4));
      const int i0 = 4 * (e % (kPairs / 4));
      const int64_t rh = (int64_t)(r_lo + rr) * kHeads + (e / (kPairs / 4)) % kHeads;
      const __nv_bfloat16* x = q + rh * kDQ + kDNope;
      const uint2 lo = *reinterpret_cast<const uint2*>(x + i0);
      const uint2 hi = *reinterpret_cast<const uint2*>(x + i0 + kPairs);
      const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
      uint32_t o1[2], o2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const double xa0 = (double)__low2float(l2[k]), xa1 = (double)__high2float(l2[k]);
        const double xb0 = (double)__low2float(h2[k]), xb1 = (double)__high2float(h2[k]);
        const double c0 = cs[rr][i0 + 2 * k][0], s0 = cs[rr][i0 + 2 * k][1];
        const double c1 = cs[rr][i0 + 2 * k + 1][0], s1 = cs[rr][i0 + 2 * k + 1][1];
        const __half2 ra = __halves2half2(__double2half(xa0 * c0 - xb0 * s0),
                                          __double2half(xa1 * c1 - xb1 * s1));
        const __half2 rb = __halves2half2(__double2half(xb0 * c0 + xa0 * s0),
                                          __double2half(xb1 * c1 + xa1 * s1));
        o1[k] = *reinterpret_cast<const uint32_t*>(&ra);
        o2[k] = *reinterpret_cast<const uint32_t*>(&rb);
      }
      __half* o = qh + rh * kDQ + kDNope;
      *reinterpret_cast<uint2*>(o + i0) = make_uint2(o1[0], o1[1]);
      *reinterpret_cast<uint2*>(o + i0 + kPairs) = make_uint2(o2[0], o2[1]);
    }
    return;
  }
  const int64_t idx = (int64_t)(blockIdx.x - q_blocks) * kPrepThreads + t;
  if (idx < ap.T * kRowPieces)
    append_piece(idx, ap.pool, ap.num_blocks, ap.block_table, ap.max_blocks, ap.batch, ap.seq_ids,
                 ap.positions, ap.c_kv, ap.k_pe, ap.status, ap.rotate, k_tab);
}

// ---------------------------------------------------------------- expand

// One CTA: 128 tokens (two cache pages) x one head.  D_K[t, d] = sum_c c_kv[t, c]
// W_UK[h][d][c] and D_V[t, v] = sum_c c_kv[t, c] W_UV[h][c][v], K = 512 latent
// dims in 4 stages of 128 through a 2-stage ring.  The A operand (the pages'
// latent columns) is K-major; W_UK[h] is K-major as stored ([d][c]) and
// W_UV[h] MN-major ([c][v]); all by TMA with the 128-byte swizzle.
constexpr int kExpThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kExpStages = 2;
constexpr uint32_t kExpStageBytes = 6 * kTile;  // A: 2 K-chunks; B_K: 2; B_V: 2 N-halves
constexpr uint32_t kExpOffBars = kExpStages * kExpStageBytes;
constexpr int kExpNumBars = 2 * kExpStages + 1;  // full, empty, done
constexpr uint32_t kExpOffTmem = kExpOffBars + 8 * kExpNumBars;
constexpr uint32_t kExpOffAbort = kExpOffTmem + 4;
constexpr uint32_t kExpSmem = kExpOffAbort + 4 + 1024;
static_assert(kExpSmem <= 232448, "shared memory per CTA");

__global__ void __launch_bounds__(kExpThreads, 1)
    kv_expand_kernel(const __grid_constant__ CUtensorMap tmap_pool,
                     const __grid_constant__ CUtensorMap tmap_wuk,
                     const __grid_constant__ CUtensorMap tmap_wuv, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  base += pad;
  auto bar = [&](int i) -> uint32_t { return base + kExpOffBars + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kExpOffAbort);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int64_t t0 = (int64_t)blockIdx.x * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kExpStages; ++s) {
      mbar_init(bar(s), 1);
      mbar_init(bar(kExpStages + s), 1);
    }
    mbar_init(bar(2 * kExpStages), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + kExpOffTmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + kExpOffTmem);
  pdl_wait();  // the chunk's rows were appended by the kernel launched before
  pdl_launch_dependents();
  int64_t seqlen = p.seqlens[b];
  if (seqlen < p.q_len || seqlen > p.max_seqlen) {
    if (threadIdx.x == 0) record_status(p.status, XMLA_ERR_DEVICE_OOB);
    seqlen = 0;
  }
  const bool active = t0 < seqlen;

  if (warp == 0) {
    if (lane == 0 && active) {
      tma_prefetch_desc(&tmap_pool);
      tma_prefetch_desc(&tmap_wuk);
      tma_prefetch_desc(&tmap_wuv);
      // the tile's two pages; a page past the sequence's end is replaced by the
      // first (its rows are never written out)
      const int64_t pg0 = t0 / kPage;
      const int64_t npages = (seqlen + kPage - 1) / kPage;
      int32_t blk[2];
      for (int k = 0; k < 2; ++k) {
        const int64_t pg = pg0 + k < npages ? pg0 + k : pg0;
        int32_t bk = p.block_table[(int64_t)b * p.max_blocks + pg];
        if (bk < 0 || (int64_t)bk >= p.num_blocks) {
          record_status(p.status, XMLA_ERR_DEVICE_OOB);
          bk = (int32_t)p.num_blocks;  // past the end: the tensor copy reads zeros
        }
        blk[k] = bk;
      }
      int issued = 0;
      for (int c = 0; c < 4; ++c) {
        const int s = c % kExpStages;
        if (c >= kExpStages &&
            !mbar_wait(bar(kExpStages + s), (uint32_t)(((c - kExpStages) / kExpStages) & 1),
                       abort_flag, p.status, p.wait_limit_ns))
          break;
        const uint32_t st = base + s * kExpStageBytes;
        mbar_arrive_expect_tx(bar(s), kExpStageBytes);
        for (int k = 0; k < 2; ++k)      // A: latent columns 128c + 64k of both pages
          for (int pg = 0; pg < 2; ++pg)
            tma_load_2d(st + k * kTile + pg * (kTile / 2), &tmap_pool, 128 * c + 64 * k,
                        blk[pg] * kPage, bar(s));
        for (int k = 0; k < 2; ++k)      // B_K: W_UK[h] rows d, columns 128c + 64k
          tma_load_2d(st + (2 + k) * kTile, &tmap_wuk, 128 * c + 64 * k, h * kDNope, bar(s));
        for (int j = 0; j < 2; ++j)      // B_V: W_UV[h] rows 128c.., v columns 64j..
          tma_load_2d(st + (4 + j) * kTile, &tmap_wuv, 64 * j, h * kDLatent + 128 * c, bar(s));
        ++issued;
      }
      for (int c = issued > kExpStages ? issued - kExpStages : 0; c < issued; ++c)
        mbar_wait(bar(c % kExpStages), (uint32_t)((c / kExpStages) & 1), nullptr, p.status,
                  p.wait_limit_ns);
    }
  } else if (warp == 1) {
    if (lane == 0 && active) {
      constexpr uint32_t idesc_k = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_v = idesc_bf16_f32(128, 128, false, true);
      bool ok = true;
      for (int c = 0; c < 4 && ok; ++c) {
        const int s = c % kExpStages;
        if (!(ok = mbar_wait(bar(s), (uint32_t)((c / kExpStages) & 1), abort_flag, p.status,
                             p.wait_limit_ns)))
          break;
        tc_fence_after();
        const uint32_t st = base + s * kExpStageBytes;
        const uint64_t a_desc = smem_desc_sw128(st, 16, 1024);
        const uint64_t bk_desc = smem_desc_sw128(st + 2 * kTile, 16, 1024);
        const uint64_t bv_desc = smem_desc_sw128(st + 4 * kTile, kTile, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // K = 128 in steps of 16
          const uint32_t kmaj = ((k >> 2) * kTile + (k & 3) * 32) >> 4;
          const uint32_t acc = (c | k) != 0 ? 1u : 0u;
          tc_mma_bf16(tmem_base, a_desc + kmaj, bk_desc + kmaj, idesc_k, acc);
          tc_mma_bf16(tmem_base + 128, a_desc + kmaj, bv_desc + ((k * 2048) >> 4), idesc_v, acc);
        }
        tc_commit(bar(kExpStages + s));
      }
      tc_commit(bar(2 * kExpStages));
    }
  } else if (active) {
    // epilogue: thread = token row; fp32 -> fp16, 256 contiguous bytes per output row;
    // rows past the sequence's end are written as zeros (the attention reads the
    // whole 128-token tile that holds the last token, and a zero probability
    // times a value read from an unwritten row could be NaN)
    const int quarter = warp & 3;
    const int64_t t = t0 + 32 * quarter + lane;
    const bool valid = active && t < seqlen;
    const int64_t row = (int64_t)b * p.s_pad + t;
    const bool ok = mbar_wait(bar(2 * kExpStages), 0, abort_flag, p.status, p.wait_limit_ns);
    tc_fence_after();
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quarter) << 16);
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {  // K_nope, then V
      __half* dst = (part == 0 ? p.kx : p.vx) + (row * kHeads + h) * 128;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(t_lane + part * 128 + 32 * cc, v);
        tc_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          w[k] = valid && ok ? pack_half2(v[2 * k], v[2 * k + 1]) : 0u;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          reinterpret_cast<uint4*>(dst + 32 * cc)[u] =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
    }
    // the rotated rope key, shared by all heads: written by the head-0 CTA of the tile
    if (h == 0) {
      uint4 o[8];
      if (valid) {
        const int32_t bk = p.block_table[(int64_t)b * p.max_blocks + t / kPage];
        const bool in = bk >= 0 && (int64_t)bk < p.num_blocks;
        const uint4* src =
            reinterpret_cast<const uint4*>(p.pool + ((int64_t)bk * kPage + t % kPage) * kDRow + kDLatent);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 x = in ? src[u] : make_uint4(0u, 0u, 0u, 0u);
          const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&x);
          o[u] = make_uint4(pack_half2(__low2float(b2[0]), __high2float(b2[0])),
                            pack_half2(__low2float(b2[1]), __high2float(b2[1])),
                            pack_half2(__low2float(b2[2]), __high2float(b2[2])),
                            pack_half2(__low2float(b2[3]), __high2float(b2[3])));
        }
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) o[u] = make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) reinterpret_cast<uint4*>(p.kp + row * kDRope)[u] = o[u];
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, 256);
  }
}

// ---------------------------------------------------------------- attend

// One CTA: 128 queries of one sequence x one head.  Tensor memory (fp32
// columns): two S buffers [128 queries x 128 tokens] at 0 and 128, O [128 x
// 128 v] at 256, and two P buffers [128 x 128 tokens] as fp16 pairs (64
// columns each) at 384 and 448, the A operand of the PV product.  Shared
// memory: Q (3 boxes of 64 dims), two K stages (K_nope: 2 boxes, rope key: 1
// box) and two V stages (2 boxes of 64 v), all by TMA with the 128-byte
// swizzle; and the row statistics the softmax warps hand on.
// Warp 0 loads Q and K, warp 10 V (each as soon as its stage is free), warp 1
// issues the MMAs, warps 2-9 are the softmax in two groups of four: group g
// (warps 2 + 4g .. 5 + 4g) takes the key tiles i = g mod 2, through S buffer g
// and P buffer g, one query row per thread (its lane of quarter warp & 3).  The
// groups overlap: while one turns its scores into probabilities, the other
// reads the next tile's; a row's running maximum passes from tile to tile
// through shared memory, so the softmax is the one-pass online form.
constexpr int kAttThreads = 352;
constexpr int kAttGroup = 128;
constexpr uint32_t kAttOffQ = 0;
constexpr uint32_t kAttOffK = kAttOffQ + 3 * kTile;
constexpr uint32_t kAttKStage = 3 * kTile;
constexpr uint32_t kAttOffV = kAttOffK + 2 * kAttKStage;
constexpr uint32_t kAttVStage = 2 * kTile;
// the running maximum handed from group to group [2][128], then each group's
// (l, m, ok) at the end [2][3][128]
constexpr uint32_t kAttOffXchg = kAttOffV + 2 * kAttVStage;
constexpr uint32_t kAttXchgBytes = (2 + 6) * 128 * 4;
constexpr uint32_t kAttOffBars = kAttOffXchg + kAttXchgBytes;
// barriers
constexpr int kBQ = 0;
constexpr int kBKFull = 1;    // 2
constexpr int kBKEmpty = 3;   // 2
constexpr int kBVFull = 5;    // 2
constexpr int kBVEmpty = 7;   // 2
constexpr int kBSFull = 9;    // 2
constexpr int kBSFree = 11;   // 2
constexpr int kBPFull = 13;   // 2
constexpr int kBPvDone = 15;  // 2
constexpr int kBDrain = 17;
constexpr int kAttNumBars = 18;
constexpr uint32_t kAttOffTmem = kAttOffBars + 8 * kAttNumBars;
constexpr uint32_t kAttOffAbort = kAttOffTmem + 4;
constexpr uint32_t kAttSmem = kAttOffAbort + 4 + 1024;
static_assert(kAttSmem <= 232448, "shared memory per CTA");
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
// a row's running maximum is raised only when a score passes it by this much
// (log2 units), so an O rescale is rare
constexpr float kAttLazyMax = 8.0f;

// The softmax waits end in __syncwarp: lanes that leave the polling loop at
// different iterations meet again before the warp-wide tcgen05.ld / st.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int* abort,
                                               int32_t* status, uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, status, limit_ns);
  __syncwarp();
  return ok;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// named barriers 1..12 among the warps of one lane quarter (64 threads: the
// one of each softmax group); the producer arrives, the consumer waits
__device__ __forceinline__ void nbar_arrive(int id) {
  asm volatile("bar.arrive %0, 64;" ::"r"(id) : "memory");
}
__device__ __forceinline__ void nbar_sync(int id) {
  asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16: A's rows are tensor-memory
// lanes, two 16-bit elements per 32-bit column (the lower K index in the low half)
__device__ __forceinline__ void tc_mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem,
                                                  uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__global__ void __launch_bounds__(kAttThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_kp,
                        const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  base += pad;
  auto bar = [&](int i) -> uint32_t { return base + kAttOffBars + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAttOffAbort);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Blocks start in the order x, y, z: every head and sequence of the last
  // query tile (the most tokens) first, then the tile before it, and so on,
  // so the long units start first across the whole grid.
  const int qt = (int)(gridDim.z - 1 - blockIdx.z);
  const int h = blockIdx.x;
  const int b = blockIdx.y;
  const int j0 = qt * 128;

  if (threadIdx.x == 0) {
    mbar_init(bar(kBQ), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBKFull + i), 1);
      mbar_init(bar(kBKEmpty + i), 1);
      mbar_init(bar(kBVFull + i), 1);
      mbar_init(bar(kBVEmpty + i), 1);
      mbar_init(bar(kBSFull + i), 1);
      mbar_init(bar(kBSFree + i), kAttGroup);
      mbar_init(bar(kBPFull + i), kAttGroup);
      mbar_init(bar(kBPvDone + i), 1);
    }
    mbar_init(bar(kBDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + kAttOffTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + kAttOffTmem);
  pdl_wait();  // Q, K, V and the rope key come from the kernels launched before
  pdl_launch_dependents();
  int64_t seqlen = p.seqlens[b];
  if (seqlen < p.q_len || seqlen > p.max_seqlen) {
    if (threadIdx.x == 0) record_status(p.status, XMLA_ERR_DEVICE_OOB);
    seqlen = 0;
  }
  const int jn = seqlen > 0 ? min(p.q_len - j0, 128) : 0;  // queries of this tile
  // key tiles: every token up to the tile's last query position
  const int nt = jn > 0 ? (int)((seqlen - p.q_len + j0 + jn - 1) / 128 + 1) : 0;
  const int64_t krow0 = (int64_t)b * p.s_pad;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nt > 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_kp);
      tma_prefetch_desc(&tmap_v);
      const int32_t qrow0 = b * p.q_len + j0;
      mbar_arrive_expect_tx(bar(kBQ), 3 * kTile);
      for (int k = 0; k < 3; ++k)
        tma_load_3d(base + kAttOffQ + k * kTile, &tmap_q, 64 * k, h, qrow0, bar(kBQ));
      // K(i) goes to stage i % 2 once QK(i - 2) is done
      int nk = 0;  // tiles whose K copies were issued
      for (int i = 0; i < nt; ++i) {
        const int s = i & 1;
        if (i >= 2 && !mbar_wait(bar(kBKEmpty + s), (uint32_t)(((i - 2) >> 1) & 1), abort_flag,
                                 p.status, p.wait_limit_ns))
          break;
        const int32_t r = (int32_t)(krow0 + 128 * (int64_t)i);
        const uint32_t kst = base + kAttOffK + s * kAttKStage;
        mbar_arrive_expect_tx(bar(kBKFull + s), kAttKStage);
        tma_load_3d(kst, &tmap_k, 0, h, r, bar(kBKFull + s));
        tma_load_3d(kst + kTile, &tmap_k, 64, h, r, bar(kBKFull + s));
        tma_load_2d(kst + 2 * kTile, &tmap_kp, 0, r, bar(kBKFull + s));
        nk = i + 1;
      }
      // every copy issued must land before the CTA may exit
      mbar_wait(bar(kBQ), 0, nullptr, p.status, p.wait_limit_ns);
      for (int i = nk > 2 ? nk - 2 : 0; i < nk; ++i)
        mbar_wait(bar(kBKFull + (i & 1)), (uint32_t)((i >> 1) & 1), nullptr, p.status,
                  p.wait_limit_ns);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ V producer
    if (lane == 0 && nt > 0) {
      // V(i) goes to stage i % 2 once PV(i - 2) is done
      int nv = 0;
      for (int i = 0; i < nt; ++i) {
        const int s = i & 1;
        if (i >= 2 && !mbar_wait(bar(kBVEmpty + s), (uint32_t)(((i - 2) >> 1) & 1), abort_flag,
                                 p.status, p.wait_limit_ns))
          break;
        const int32_t r = (int32_t)(krow0 + 128 * (int64_t)i);
        const uint32_t vst = base + kAttOffV + s * kAttVStage;
        mbar_arrive_expect_tx(bar(kBVFull + s), kAttVStage);
        tma_load_3d(vst, &tmap_v, 0, h, r, bar(kBVFull + s));
        tma_load_3d(vst + kTile, &tmap_v, 64, h, r, bar(kBVFull + s));
        nv = i + 1;
      }
      for (int i = nv > 2 ? nv - 2 : 0; i < nv; ++i)
        mbar_wait(bar(kBVFull + (i & 1)), (uint32_t)((i >> 1) & 1), nullptr, p.status,
                  p.wait_limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nt > 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, 128, false, true);
      const uint64_t d_q = smem_desc_sw128(base + kAttOffQ, 16, 1024);
      const uint64_t d_k = smem_desc_sw128(base + kAttOffK, 16, 1024);
      const uint64_t d_v = smem_desc_sw128(base + kAttOffV, kTile, 1024);
      auto wait = [&](int idx, uint32_t parity) {
        return mbar_wait(bar(idx), parity, abort_flag, p.status, p.wait_limit_ns);
      };
      auto qk = [&](int i) {
        const int s = i & 1;
        if (!wait(kBKFull + s, (uint32_t)((i >> 1) & 1))) return false;
        if (i >= 2 && !wait(kBSFree + s, (uint32_t)(((i - 2) >> 1) & 1))) return false;
        tc_fence_after();
        const uint64_t bk = d_k + ((s * kAttKStage) >> 4);
#pragma unroll
        for (int k = 0; k < 12; ++k) {  // K = 192 in steps of 16
          const uint32_t off = ((k >> 2) * kTile + (k & 3) * 32) >> 4;
          tc_mma_f16(tmem_base + kColS + 128 * s, d_q + off, bk + off, idesc_qk, k != 0 ? 1u : 0u);
        }
        tc_commit(bar(kBKEmpty + s));
        tc_commit(bar(kBSFull + s));
        return true;
      };
      bool ok = wait(kBQ, 0);
      tc_fence_after();
      if (ok) ok = qk(0);
      if (ok && nt > 1) ok = qk(1);
      for (int i = 0; i < nt && ok; ++i) {
        // QK(i + 2) first: its S buffer is free as soon as tile i's scores are read
        if (i + 2 < nt && !(ok = qk(i + 2))) break;
        const int s = i & 1;
        if (!(ok = wait(kBPFull + s, (uint32_t)((i >> 1) & 1)))) break;
        if (!(ok = wait(kBVFull + s, (uint32_t)((i >> 1) & 1)))) break;
        tc_fence_after();
        const uint64_t bv = d_v + ((s * kAttVStage) >> 4);
#pragma unroll
        for (int k = 0; k < 8; ++k)  // K = 128 tokens in steps of 16 (8 columns of P)
          tc_mma_f16_tmem_a(tmem_base + kColO, tmem_base + kColP + 64 * s + 8 * k,
                            bv + ((k * 2048) >> 4), idesc_pv, (i | k) != 0 ? 1u : 0u);
        tc_commit(bar(kBVEmpty + s));
        tc_commit(bar(kBPvDone + s));
      }
      tc_commit(bar(kBDrain));
      mbar_wait(bar(kBDrain), 0, nullptr, p.status, p.wait_limit_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax, one query row per thread
    const int g = (warp - 2) >> 2;        // key tiles i = g mod 2
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;  // tensor-memory lane = query row of the tile
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quarter) << 16);
    float* hand = reinterpret_cast<float*>(smem + kAttOffXchg);  // [from group][row]
    float* fin = hand + 2 * 128;                                // [group][l, m, ok][row]
    const int j = j0 + row;
    // the row's last visible token (the query's own position); -1 for a padding row
    const int64_t qpos = j < j0 + jn ? seqlen - p.q_len + j : -1;
    // tiles from here on hold tokens past some row's position: they are masked
    const int64_t first_masked = (seqlen - p.q_len + j0 + 1) / 128;
    const float sc = p.scale_log2;
    // m_w: the running maximum (log2 units) this group's l_w is expressed in
    float l_w = 0.f, m_w = -INFINITY;
    bool ok = true;
    // No exit before the end: every handoff below has its partner in the other
    // group, so a failed wait only marks the thread, which carries on with
    // whatever it read (the abort flag makes the remaining waits short).
    for (int i = g; i < nt; i += 2) {
      ok &= mbar_wait_warp(bar(kBSFull + g), (uint32_t)((i >> 1) & 1), abort_flag, p.status,
                      p.wait_limit_ns);
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float (&xc)[32] = *reinterpret_cast<float(*)[32]>(x + 32 * c);
        tmem_ld32(t_lane + kColS + 128 * g + 32 * c, xc);
      }
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(kBSFree + g));
      if (i >= first_masked) {
        const int64_t lim64 = qpos - 128 * (int64_t)i;
        const int lim = lim64 < -1 ? -1 : (lim64 > 128 ? 128 : (int)lim64);
#pragma unroll
        for (int k = 0; k < 128; ++k) x[k] = k <= lim ? x[k] : -INFINITY;
      }
      float mxs;
      {
        float t[16];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          t[u] = fmax3(fmax3(x[8 * u], x[8 * u + 1], x[8 * u + 2]),
                       fmax3(x[8 * u + 3], x[8 * u + 4], x[8 * u + 5]), fmaxf(x[8 * u + 6], x[8 * u + 7]));
        const float a = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]), fmax3(t[6], t[7], t[8]));
        const float b2 = fmax3(fmax3(t[9], t[10], t[11]), fmax3(t[12], t[13], t[14]), t[15]);
        mxs = fmaxf(a, b2) * sc;  // in log2 units
      }
      // the running maximum after tile i - 1, from the other group
      float m_prev = -INFINITY;
      if (i >= 1) {
        nbar_sync(1 + 4 * (g ^ 1) + quarter);
        m_prev = hand[(g ^ 1) * 128 + row];
      }
      const bool raise = mxs > m_prev + kAttLazyMax;
      const float m_cur = raise ? mxs : m_prev;
      if (i + 1 < nt) {
        hand[g * 128 + row] = m_cur;
        nbar_arrive(1 + 4 * g + quarter);
      }
      if (i >= 1 && __any_sync(0xffffffffu, raise)) {
        // O holds PV(i - 1) once that product completes; the warp rescales its
        // rows together (tensor-memory access is per warp)
        ok &= mbar_wait_warp(bar(kBPvDone + (g ^ 1)), (uint32_t)(((i - 1) >> 1) & 1), abort_flag,
                        p.status, p.wait_limit_ns);
        tc_fence_after();
        const float f = raise && m_prev != -INFINITY ? ex2(m_prev - m_cur) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(t_lane + kColO + 32 * c, o);
          tc_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= f;
          tmem_st32(t_lane + kColO + 32 * c, o);
        }
      }
      if (m_cur != m_w) {
        l_w = m_w == -INFINITY ? 0.f : l_w * ex2(m_w - m_cur);
        m_w = m_cur;
      }
      // P buffer g was read by PV(i - 2)
      if (i >= 2)
        ok &= mbar_wait_warp(bar(kBPvDone + g), (uint32_t)(((i - 2) >> 1) & 1), abort_flag, p.status,
                        p.wait_limit_ns);
      tc_fence_after();
      // probabilities as fp16 pairs (token 2w in the low half of column w) into
      // the row's 64 columns of P buffer g; l sums them before the rounding
      const float msub = m_cur == -INFINITY ? 0.f : m_cur;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2(fmaf(x[64 * c + 2 * e], sc, -msub));
          const float p1 = ex2(fmaf(x[64 * c + 2 * e + 1], sc, -msub));
          ls[e & 3] += p0 + p1;
          const __half2 hv = __floats2half2_rn(p0, p1);
          w[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        tmem_st32u(t_lane + kColP + 64 * g + 32 * c, w);
      }
      l_w += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBPFull + g));
    }
    // ---- epilogue: the groups' sums brought to the final maximum; O / l as the
    // bf16 output row of (query, head), v columns 64 g .. 64 g + 63 by group g
    if (nt > 0)
      ok &= mbar_wait_warp(bar(kBPvDone + ((nt - 1) & 1)), (uint32_t)(((nt - 1) >> 1) & 1), abort_flag,
                      p.status, p.wait_limit_ns);
    fin[(3 * g + 0) * 128 + row] = l_w;
    fin[(3 * g + 1) * 128 + row] = m_w;
    fin[(3 * g + 2) * 128 + row] = ok ? 1.f : 0.f;
    nbar_sync(9 + quarter);
    const float l_o = fin[(3 * (g ^ 1) + 0) * 128 + row];
    const float m_o = fin[(3 * (g ^ 1) + 1) * 128 + row];
    const bool have = nt > 0 && ok && fin[(3 * (g ^ 1) + 2) * 128 + row] != 0.f;
    if (!__any_sync(0xffffffffu, !have)) {
      tc_fence_after();
      const float m_f = fmaxf(m_w, m_o);
      float lt = 0.f;
      if (m_w != -INFINITY) lt += l_w * ex2(m_w - m_f);
      if (m_o != -INFINITY) lt += l_o * ex2(m_o - m_f);
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      __nv_bfloat16* dst = p.out + ((int64_t)(b * p.q_len + j) * kHeads + h) * kDV + 64 * g;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float o[32];
        tmem_ld32(t_lane + kColO + 64 * g + 32 * c, o);
        tc_wait_ld();
        if (qpos >= 0) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 v =
                  __floats2bfloat162_rn(o[8 * u + 2 * e] * inv, o[8 * u + 2 * e + 1] * inv);
              wv[e] = *reinterpret_cast<const uint32_t*>(&v);
            }
            reinterpret_cast<uint4*>(dst + 32 * c)[u] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, 512);
  }
}

template <typename Kern>
static cudaError_t set_smem(Kern k, uint32_t bytes, bool* done) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_prefill_prep(const __nv_bfloat16* q, const int32_t* seqlens, __half* qh, int rows,
                                int q_len, const RopeTable& q_tab, const AppendArgs& ap,
                                const RopeTable& k_tab, cudaStream_t st) {
  const int64_t q_blocks = (rows + kPrepRows - 1) / kPrepRows;
  const int64_t a_blocks = (ap.T * kRowPieces + kPrepThreads - 1) / kPrepThreads;
  if (q_blocks + a_blocks > (1 << 30)) return cudaErrorInvalidValue;
  return launch_pdl(prefill_prep_kernel, dim3((unsigned)(q_blocks + a_blocks)), dim3(kPrepThreads),
                    0, st, q, seqlens, qh, rows, q_len, q_tab, ap, k_tab);
}

cudaError_t launch_kv_expand(const CUtensorMap& pool_map, const CUtensorMap& wuk_map,
                             const CUtensorMap& wuv_map, const PrefillParams& p, cudaStream_t st) {
  static bool done[64] = {};
  const cudaError_t e = set_smem(kv_expand_kernel, kExpSmem, done);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(p.s_pad / 128), kHeads, (unsigned)p.batch);
  return launch_pdl(kv_expand_kernel, grid, dim3(kExpThreads), kExpSmem, st, pool_map, wuk_map,
                    wuv_map, p);
}

cudaError_t launch_prefill_attn(const CUtensorMap& q_map, const CUtensorMap& k_map,
                                const CUtensorMap& kp_map, const CUtensorMap& v_map,
                                const PrefillParams& p, cudaStream_t st) {
  static bool done[64] = {};
  const cudaError_t e = set_smem(prefill_attn_kernel, kAttSmem, done);
  if (e != cudaSuccess) return e;
  const dim3 grid(kHeads, (unsigned)p.batch, (unsigned)((p.q_len + 127) / 128));
  return launch_pdl(prefill_attn_kernel, grid, dim3(kAttThreads), kAttSmem, st, q_map, k_map,
                    kp_map, v_map, p);
}

}  // namespace xmla
