// Per-head products of a long query batch (a prompt chunk) on the tensor cores.
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": kv_b_proj maps the 512-dim latent to 32 heads x (128 K_nope +
//      128 V); in the absorbed form its K half (W_UK) multiplies the query and its
//      V half (W_UV) the probability-weighted latent sum.
//
// With a few query rows these are small per-head matrix-vector products (the
// absorb and combine kernels do them on the CUDA cores).  A prompt chunk has
// thousands of rows, and both become per-head GEMMs of 17 GFLOP for 4096 rows:
//   absorb:  q_lat[r, h, :] = q_nope[r, h, :] . W_UK[h]        [R x 128] x [128 x 512]
//   W_UV:    out[r, h, :]   = o_lat[r, h, :] . W_UV[h]         [R x 512] x [512 x 128]
// One CTA computes a 128-row tile of one head with tcgen05 (fp32 accumulators in
// tensor memory).  The A operand comes K-major (rows of the query or of o_lat),
// the B operand MN-major (W_UK[h] and W_UV[h] as stored), both by TMA with the
// 128-byte swizzle.  The W_UV product takes o_lat as two bf16 parts, hi and lo =
// bf16(o_lat - hi), accumulated into the same tile, so it carries ~16 bits of
// o_lat; the absorb writes its fp32 result as the split-K kernel's hi/lo query.
#include <cuda.h>

#include <cstdint>

#include "decode_chain.h"

namespace xmla {

namespace {

constexpr int kGemmRows = 128;     // M: query rows per CTA
constexpr int kGemmThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t kBox = 16384;   // one 128 x 64 bf16 box (128-byte rows)

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int32_t x, int32_t y,
                                            int32_t z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// Shared memory: the absorb holds its whole K = 128 at once (A: 2 boxes, B: 4
// boxes of 64 latent columns); the W_UV product streams K = 512 in 4 chunks of
// 128 through 2 stages (A hi: 2 boxes, A lo: 2 boxes, B: 2 boxes of 64 v).
template <bool kAbsorb>
struct GemmLayout {
  static constexpr int kStages = kAbsorb ? 1 : 2;
  static constexpr int kChunks = kAbsorb ? 1 : 4;
  static constexpr uint32_t kStageBytes = kAbsorb ? 6 * kBox : 6 * kBox;
  static constexpr int kN = kAbsorb ? 256 : 128;  // accumulator columns
  static constexpr uint32_t kOffBars = kStages * kStageBytes;
  // barriers: full[kStages], empty[kStages], done
  static constexpr int kNumBars = 2 * kStages + 1;
  static constexpr uint32_t kOffTmem = kOffBars + 8 * kNumBars;
  static constexpr uint32_t kOffAbort = kOffTmem + 4;
  static constexpr uint32_t kSmem = kOffAbort + 4 + 1024;  // slack for 1024-byte alignment
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

// The two products.  tmap_a: the query [R, 32, 192] (absorb) or o_lat hi
// [R, 32, 512]; tmap_a2: o_lat lo (W_UV only); tmap_b: W_UK as [32 * 128, 512]
// or W_UV as [32 * 512, 128].  Grid: (row tiles, 32 heads, 2 column halves for
// the absorb / 1).
template <bool kAbsorb>
__global__ void __launch_bounds__(kGemmThreads, 1)
    head_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_a2,
                     const __grid_constant__ CUtensorMap tmap_b, const HeadGemmParams p) {
  using L = GemmLayout<kAbsorb>;
  extern __shared__ uint8_t smem_raw[];
  uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  base += pad;
  auto bar = [&](int i) -> uint32_t { return base + L::kOffBars + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * kGemmRows;
  const int h = blockIdx.y;
  const int n0 = blockIdx.z * L::kN;  // first output column of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(s), 1);
      mbar_init(bar(L::kStages + s), 1);
    }
    mbar_init(bar(2 * L::kStages), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::kOffTmem, L::kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
      if (!kAbsorb) tma_prefetch_desc(&tmap_a2);
      // the query, o_lat and the weights may come from the kernels launched before
      pdl_wait();
      int issued = 0;
      for (int c = 0; c < L::kChunks; ++c) {
        const int s = c % L::kStages;
        if (c >= L::kStages &&
            !mbar_wait(bar(L::kStages + s), (uint32_t)(((c - L::kStages) / L::kStages) & 1),
                       abort_flag, p.status, p.wait_limit_ns))
          break;
        const uint32_t st = base + s * L::kStageBytes;
        mbar_arrive_expect_tx(bar(s), L::kStageBytes);
        if constexpr (kAbsorb) {
          // A: q_nope columns 0..127 of head h, rows r0..r0+127
          tma_load_3d(st, &tmap_a, 0, h, r0, bar(s));
          tma_load_3d(st + kBox, &tmap_a, 64, h, r0, bar(s));
          // B: W_UK[h] rows d = 0..127, latent columns n0..n0+255 in 4 boxes of 64
          for (int j = 0; j < 4; ++j)
            tma_load_2d(st + (2 + j) * kBox, &tmap_b, n0 + 64 * j, h * 128, bar(s));
        } else {
          const int k0 = 128 * c;  // latent columns of this chunk
          tma_load_3d(st, &tmap_a, k0, h, r0, bar(s));
          tma_load_3d(st + kBox, &tmap_a, k0 + 64, h, r0, bar(s));
          tma_load_3d(st + 2 * kBox, &tmap_a2, k0, h, r0, bar(s));
          tma_load_3d(st + 3 * kBox, &tmap_a2, k0 + 64, h, r0, bar(s));
          // B: W_UV[h] rows c = k0..k0+127, v columns in 2 boxes of 64
          for (int j = 0; j < 2; ++j)
            tma_load_2d(st + (4 + j) * kBox, &tmap_b, 64 * j, h * 512 + k0, bar(s));
        }
        ++issued;
      }
      // every copy issued must land before the CTA may exit
      for (int c = issued > L::kStages ? issued - L::kStages : 0; c < issued; ++c)
        mbar_wait(bar(c % L::kStages), (uint32_t)((c / L::kStages) & 1), nullptr, p.status,
                  p.wait_limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGemmRows, L::kN, false, true);
      bool ok = true;
      for (int c = 0; c < L::kChunks && ok; ++c) {
        const int s = c % L::kStages;
        if (!(ok = mbar_wait(bar(s), (uint32_t)((c / L::kStages) & 1), abort_flag, p.status,
                             p.wait_limit_ns)))
          break;
        tc_fence_after();
        const uint32_t st = base + s * L::kStageBytes;
        // A K-major (rows of 128 B, 8-row groups 1024 B apart); B MN-major (a row of
        // 64 N values per K index, 8-row K groups 1024 B apart, N groups one box apart)
        const uint32_t b_off = kAbsorb ? 2 * kBox : 4 * kBox;
        const uint64_t b_desc = smem_desc_sw128(st + b_off, kBox, 1024);
        const int parts = kAbsorb ? 1 : 2;  // hi, lo
        for (int part = 0; part < parts; ++part) {
          const uint64_t a_desc = smem_desc_sw128(st + part * 2 * kBox, 16, 1024);
#pragma unroll
          for (int k = 0; k < 8; ++k) {  // K = 128 in steps of 16
            const uint64_t a = a_desc + (((k >> 2) * kBox + (k & 3) * 32) >> 4);
            const uint64_t b = b_desc + ((k * 2048) >> 4);
            tc_mma_bf16(tmem_base, a, b, idesc, (c | part | k) != 0 ? 1u : 0u);
          }
        }
        tc_commit(bar(L::kStages + s));  // the stage may be refilled
      }
      // the accumulator is complete (after a timeout: every MMA that was issued)
      tc_commit(bar(2 * L::kStages));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each thread converts its row's 32 columns of a column block; the warp
    // passes them through a private staging tile in the (now idle) operand
    // stages, so that every global store writes 64 contiguous bytes of a row
    // (8 rows x 4 lanes per instruction) instead of 16 bytes in 32 rows.
    const int quarter = warp & 3;
    const bool ok = mbar_wait(bar(2 * L::kStages), 0, abort_flag, p.status, p.wait_limit_ns);
    tc_fence_after();
    const uint32_t t_lane = tmem_base + ((uint32_t)(32 * quarter) << 16);
    constexpr uint32_t kStgRow = 80;                   // 64 B of a row + 16 B of padding
    constexpr uint32_t kStgPart = 32 * kStgRow;
    uint8_t* stg = smem + quarter * 2 * kStgPart;      // [part][32 rows][80 B]
    const int srow = lane >> 2, piece = lane & 3;  // staging row (+ 8 j) and 16-byte piece
#pragma unroll 1
    for (int cc = 0; cc < L::kN / 32; ++cc) {
      float v[32];
      tmem_ld32(t_lane + 32 * cc, v);
      tc_wait_ld();
      if (!__all_sync(0xffffffffu, ok && *abort_flag == 0)) continue;
      uint32_t w0[16], w1[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if constexpr (kAbsorb) {
          const float a = v[2 * k] * p.scale, b = v[2 * k + 1] * p.scale;
          const __nv_bfloat162 hv = __floats2bfloat162_rn(a, b);
          const __nv_bfloat162 lv =
              __floats2bfloat162_rn(a - __low2float(hv), b - __high2float(hv));
          w0[k] = *reinterpret_cast<const uint32_t*>(&hv);
          w1[k] = *reinterpret_cast<const uint32_t*>(&lv);
        } else {
          const __nv_bfloat162 ov = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
          w0[k] = *reinterpret_cast<const uint32_t*>(&ov);
          w1[k] = 0u;
        }
      }
      constexpr int kParts = kAbsorb ? 2 : 1;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        *reinterpret_cast<uint4*>(stg + lane * kStgRow + 16 * u) =
            make_uint4(w0[4 * u], w0[4 * u + 1], w0[4 * u + 2], w0[4 * u + 3]);
        if constexpr (kParts == 2)
          *reinterpret_cast<uint4*>(stg + kStgPart + lane * kStgRow + 16 * u) =
              make_uint4(w1[4 * u], w1[4 * u + 1], w1[4 * u + 2], w1[4 * u + 3]);
      }
      __syncwarp();
#pragma unroll
      for (int part = 0; part < kParts; ++part) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int rr = srow + 8 * j;
          const int grow = r0 + 32 * quarter + rr;
          if (grow < p.rows) {
            const uint4 val =
                *reinterpret_cast<const uint4*>(stg + part * kStgPart + rr * kStgRow + 16 * piece);
            if constexpr (kAbsorb) {
              // q_ext rows: the 32 heads' hi parts of query row r, then their lo parts
              *reinterpret_cast<uint4*>(p.q_ext + ((int64_t)(2 * grow + part) * kHeads + h) * kDRow +
                                        n0 + 32 * cc + 8 * piece) = val;
            } else {
              *reinterpret_cast<uint4*>(p.out + ((int64_t)grow * kHeads + h) * kDV + 32 * cc +
                                        8 * piece) = val;
            }
          }
        }
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, L::kN);
  }
}

}  // namespace

template <bool kAbsorb>
static cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& ta2, const CUtensorMap& tb,
                               const HeadGemmParams& p, cudaStream_t st) {
  using L = GemmLayout<kAbsorb>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(head_gemm_kernel<kAbsorb>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)((p.rows + kGemmRows - 1) / kGemmRows), kHeads, kAbsorb ? 2 : 1);
  return launch_pdl(head_gemm_kernel<kAbsorb>, grid, dim3(kGemmThreads), L::kSmem, st, ta, ta2, tb,
                    p);
}

cudaError_t launch_absorb_gemm(const CUtensorMap& q_map, const CUtensorMap& wuk_map,
                               const HeadGemmParams& p, cudaStream_t st) {
  return launch_gemm<true>(q_map, q_map, wuk_map, p, st);
}

cudaError_t launch_uv_gemm(const CUtensorMap& ohi_map, const CUtensorMap& olo_map,
                           const CUtensorMap& wuv_map, const HeadGemmParams& p, cudaStream_t st) {
  return launch_gemm<false>(ohi_map, olo_map, wuv_map, p, st);
}

}  // namespace xmla
