// The two small kernels around the split-K attention of a decode call:
// q absorb (optionally fused with the step's cache append) before it, and the
// split merge with the W_UV product after it.
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": kv_b_proj maps the 512-dim latent to 32 heads x (128 K_nope +
//      128 V); the absorbed form applies its K half (W_UK) to the query and its V
//      half (W_UV) to the probability-weighted latent sum.
// [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 一: q_pe
//      is rotated by YaRN RoPE at the query's position.
#include <cooperative_groups.h>

#include <cmath>
#include <cstdint>

#include "append.cuh"
#include "decode_chain.h"
#include "produce.cuh"

namespace cg = cooperative_groups;

namespace xmla {

// ---------------------------------------------------------------- q absorb

// q_ext[r, h] = qscale * [W_UK[h]^T q_nope[r, h] | rope(q_pe[r, h], pos_r)], r = b*q_len + j,
// with pos_r = seqlens[b] - q_len + j (the q_len new tokens are the last cache
// entries).  Blocks (32 heads x 8 blocks of 64 latent columns) of 128 threads:
// thread t owns 8 columns (t % 8) and 8 of the 128 nope dims (t / 8), holding
// its 8 x 8 slice of W_UK in registers (loaded before the wait on the kernel
// launched just before, which it does not depend on); partial sums meet in
// shared memory.  A ninth block per head rotates the rope part.
constexpr int kAbsorbRows = 8;
constexpr int kAbsorbThreads = 128;
constexpr int kAbsorbBlocks = kHeads * (kDLatent / 64 + 1);

// Shared memory of one absorb block: q_nope rows and the per-thread-group sums.
struct AbsorbSmem {
  float sq[kAbsorbRows][kDNope];
  float part[16][kAbsorbRows][64];
};

// Row of q_ext holding head h of query row r (r = b*q_len + j): split, each
// row group of 32 heads is followed by its low halves (part 1), q = hi + lo
// with hi = bf16(q) and lo = bf16(q - hi); otherwise one bf16 row.
__device__ __forceinline__ int64_t q_ext_row(int64_t r, int h, int part, int split) {
  return split ? (2 * r + part) * kHeads + h : r * kHeads + h;
}

// Block (h, cb) of the absorb; cb == 8 is the rope block.  Every block waits
// (griddepcontrol.wait) before reading q or seqlens: a preceding kernel may
// have written them, and the split-K kernel relies on that wait (its producer
// reads cache rows appended by the kernel before this one).
// kF16: q_ext rows hold f16 values (one row per query row; split unused).
template <bool kRowBlocks, bool kF16 = false>
__device__ __forceinline__ void q_absorb_block(int h, int cb, const __nv_bfloat16* q,
                                               const __nv_bfloat16* __restrict__ W_UK,
                                               const int32_t* seqlens,
                                               __nv_bfloat16* __restrict__ q_ext, int rows,
                                               int q_len, int split, float qscale,
                                               const RopeTable& tab, AbsorbSmem& sm,
                                               int row_lo_arg, int row_hi_arg) {
  // kRowBlocks: rows [row_lo, row_hi) of the query; otherwise all rows
  const int row_lo = kRowBlocks ? row_lo_arg : 0;
  const int row_hi = kRowBlocks ? row_hi_arg : rows;
  auto& sq = sm.sq;
  auto& part = sm.part;
  const int t = threadIdx.x;
  if (cb == kDLatent / 64) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int kPairs = kDRope / 2;
    for (int e = row_lo * kPairs + t; e < row_hi * kPairs; e += kAbsorbThreads) {
      const int r = e / kPairs, i = e % kPairs;
      const int64_t pos = (int64_t)seqlens[r / q_len] - q_len + (r % q_len);
      const __nv_bfloat16* x = q + ((int64_t)r * kHeads + h) * kDQ + kDNope;
      double y1, y2;
      rope_pair((double)__bfloat162float(x[i]), (double)__bfloat162float(x[i + kPairs]), pos, i,
                tab, &y1, &y2);
      const double v1 = y1 * (double)qscale, v2 = y2 * (double)qscale;
      if constexpr (kF16) {
        __half* o = reinterpret_cast<__half*>(q_ext) + ((int64_t)r * kHeads + h) * kDRow + kDLatent;
        o[i] = __double2half(v1);
        o[i + kPairs] = __double2half(v2);
        continue;
      }
      const __nv_bfloat16 h1 = __double2bfloat16(v1), h2 = __double2bfloat16(v2);
      __nv_bfloat16* o = q_ext + q_ext_row(r, h, 0, split) * kDRow + kDLatent;
      o[i] = h1;
      o[i + kPairs] = h2;
      if (split) {  // the low halves, one block of 32 rows further
        __nv_bfloat16* ol = q_ext + q_ext_row(r, h, 1, split) * kDRow + kDLatent;
        ol[i] = __double2bfloat16(v1 - (double)__bfloat162float(h1));
        ol[i + kPairs] = __double2bfloat16(v2 - (double)__bfloat162float(h2));
      }
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
  pdl_launch_dependents();
  for (int r0 = row_lo; r0 < row_hi; r0 += kAbsorbRows) {
    const int nr = min(kAbsorbRows, row_hi - r0);
    __syncthreads();
    for (int e = t; e < nr * kDNope; e += kAbsorbThreads) {
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
    for (int o = t; o < nr * 64; o += kAbsorbThreads) {
      const int r = o / 64, col = o % 64;
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) s += part[k][r][col];
      const float v = s * qscale;
      if constexpr (kF16) {
        reinterpret_cast<__half*>(q_ext)[((int64_t)(r0 + r) * kHeads + h) * kDRow + cb * 64 + col] =
            __float2half_rn(v);
        continue;
      }
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      q_ext[q_ext_row(r0 + r, h, 0, split) * kDRow + cb * 64 + col] = hi;
      if (split)
        q_ext[q_ext_row(r0 + r, h, 1, split) * kDRow + cb * 64 + col] =
            __float2bfloat16_rn(v - __bfloat162float(hi));
    }
  }
}

// Rope columns of q_ext for the rows [r_lo, r_hi) (at most kRopeRows) of all 32
// heads, for a prompt chunk whose latent columns come from the tensor-core
// absorb.  The rotation angle depends only on the position and the pair, so the
// block forms cos and sin once per (row, pair) -- float64, the same arithmetic as
// rope_pair -- and applies them to every head.
__device__ __forceinline__ void q_rope_rows_block(int r_lo, int r_hi, const __nv_bfloat16* q,
                                                  const int32_t* seqlens,
                                                  __nv_bfloat16* __restrict__ q_ext, int q_len,
                                                  int split, float qscale, const RopeTable& tab,
                                                  AbsorbSmem& sm) {
  constexpr int kPairs = kDRope / 2;
  static_assert(sizeof(sm.sq) >= 2 * sizeof(double) * 4 * kPairs, "cos/sin table");
  double* cs = reinterpret_cast<double*>(&sm.sq[0][0]);  // [row][pair] (cos, sin)
  const int t = threadIdx.x;
  const int nr = r_hi - r_lo;
  pdl_wait();
  pdl_launch_dependents();
  if (t < nr * kPairs) {
    const int r = r_lo + t / kPairs, i = t % kPairs;
    const int64_t pos = (int64_t)seqlens[r / q_len] - q_len + (r % q_len);
    double sn, c;
    sincos((double)pos * tab.inv_freq[i], &sn, &c);
    cs[2 * t] = c * tab.magnitude;
    cs[2 * t + 1] = sn * tab.magnitude;
  }
  __syncthreads();
  for (int e = t; e < nr * kHeads * kPairs; e += kAbsorbThreads) {
    const int rr = e / (kHeads * kPairs), h = (e / kPairs) % kHeads, i = e % kPairs;
    const int r = r_lo + rr;
    const double c = cs[2 * (rr * kPairs + i)], sn = cs[2 * (rr * kPairs + i) + 1];
    const __nv_bfloat16* x = q + ((int64_t)r * kHeads + h) * kDQ + kDNope;
    const double x1 = (double)__bfloat162float(x[i]), x2 = (double)__bfloat162float(x[i + kPairs]);
    const double v1 = (x1 * c - x2 * sn) * (double)qscale;
    const double v2 = (x2 * c + x1 * sn) * (double)qscale;
    const __nv_bfloat16 h1 = __double2bfloat16(v1), h2 = __double2bfloat16(v2);
    __nv_bfloat16* o = q_ext + q_ext_row(r, h, 0, split) * kDRow + kDLatent;
    o[i] = h1;
    o[i + kPairs] = h2;
    if (split) {
      __nv_bfloat16* ol = q_ext + q_ext_row(r, h, 1, split) * kDRow + kDLatent;
      ol[i] = __double2bfloat16(v1 - (double)__bfloat162float(h1));
      ol[i + kPairs] = __double2bfloat16(v2 - (double)__bfloat162float(h2));
    }
  }
}

// ---------------------------------------------------------------- length-aware split plan

// Sum (kMax false) or maximum over the 128 threads of a block, returned to all.
template <bool kMax>
__device__ __forceinline__ long long plan_reduce(long long v, long long* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const long long x = __shfl_xor_sync(0xffffffffu, v, o);
    v = kMax ? max(v, x) : v + x;
  }
  __syncthreads();  // the previous call's readers are done with red
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int k = 1; k < kAbsorbThreads / 32; ++k) v = kMax ? max(v, red[k]) : v + red[k];
  return v;
}

// Shared memory of the plan kernel: pages per unit, reduction and scan slots.
struct PlanSmem {
  int w[kMaxPlanCtas];
  long long red[kAbsorbThreads / 32];
  int scan[kAbsorbThreads / 32];
};

// The plan of WorkPlanArgs, by one block of 128 threads.  Unit u = b * groups
// + g has w_u = ceil(seqlen_b / 64) pages; T is the smallest page count per
// CTA for which sum_u max(1, ceil(w_u / T)) CTAs fit in the grid (at least two
// pages per CTA unless a unit has fewer), found by bisection: T = ceil(total /
// (ctas - units)) always fits, and so does T = max_u w_u.  Unit u then gets
// ns_u = max(1, ceil(w_u / T)) CTAs, consecutive in unit order, each a run of
// ceil(w_u / ns_u) <= T pages; CTAs past the last unit get no work.  It runs
// as one extra block of the first kernel of a decode call, side by side with
// the absorb; the split-K kernel waits for that kernel and so finds the tables.
__device__ __forceinline__ void work_plan_block(const WorkPlanArgs& a, PlanSmem& sm) {
  int* w_s = sm.w;
  long long* red = sm.red;
  int* scan_s = sm.scan;
  const int t = threadIdx.x;
  const int units = a.batch * a.groups;  // < a.ctas <= kMaxPlanCtas = 2 * kAbsorbThreads
  pdl_wait();                            // the lengths may come from the kernel launched before
  pdl_launch_dependents();
  long long tot = 0, wmax = 0;
  // w_s[u]: the unit's cost in pages (short units of the mixed kernel take one
  // pass per query of the row group)
  for (int u = t; u < units; u += kAbsorbThreads) {
    int64_t n = a.seqlens[u / a.groups];
    if (n < 0 || n > a.max_seqlen) n = 0;  // the split-K kernel reports the bad length
    int w = (int)((n + kPage - 1) / kPage);
    if (w <= a.short_pages) w *= a.short_weight;
    w_s[u] = w;
    tot += w;
    wmax = max(wmax, (long long)w);
  }
  tot = plan_reduce<false>(tot, red);
  wmax = plan_reduce<true>(wmax, red);
  const long long spare = a.ctas - units;
  long long lo = max(max(1LL, (tot + a.ctas - 1) / a.ctas), min(2LL, wmax));
  long long hi = max(lo, min(max(wmax, 1LL), max(1LL, (tot + spare - 1) / spare)));
  while (lo < hi) {  // uniform across the block: every thread sees the same sums
    const long long mid = (lo + hi) >> 1;
    long long c = 0;
    for (int u = t; u < units; u += kAbsorbThreads) c += max(1LL, (w_s[u] + mid - 1) / mid);
    c = plan_reduce<false>(c, red);
    if (c <= a.ctas) hi = mid;
    else lo = mid + 1;
  }
  const long long T = lo;
  // first CTA of each unit: exclusive prefix sum of ns_u, units 2t and 2t + 1 on thread t
  const int u0 = 2 * t, u1 = 2 * t + 1;
  const int ns0 = u0 < units ? (int)max(1LL, (w_s[u0] + T - 1) / T) : 0;
  const int ns1 = u1 < units ? (int)max(1LL, (w_s[u1] + T - 1) / T) : 0;
  const int v = ns0 + ns1;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if ((t & 31) >= o) incl += x;
  }
  if ((t & 31) == 31) scan_s[t >> 5] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int k = 0; k < kAbsorbThreads / 32; ++k) {
    before += k < (t >> 5) ? scan_s[k] : 0;
    total += scan_s[k];
  }
  const int first0 = before + incl - v;
  auto emit = [&](int u, int first, int ns) {
    int64_t n = a.seqlens[u / a.groups];  // the unit's pages, unweighted
    if (n < 0 || n > a.max_seqlen) n = 0;
    const int w = (int)((n + kPage - 1) / kPage);
    const int pps = (w + ns - 1) / ns;
    a.unit_tab[u] = make_int2(first, ns);
    for (int s = 0; s < ns; ++s)
      a.work_tab[first + s] = make_int4(u, min(w, s * pps), min(w, (s + 1) * pps), 0);
  };
  if (ns0 > 0) emit(u0, first0, ns0);
  if (ns1 > 0) emit(u1, first0 + ns0, ns1);
  for (int k = total + t; k < a.ctas; k += kAbsorbThreads) a.work_tab[k] = make_int4(-1, 0, 0, 0);
}

static bool plan_ok(const WorkPlanArgs& plan) {
  return plan.ctas > plan.batch * plan.groups && plan.ctas <= kMaxPlanCtas;
}

// q and seqlens carry no __restrict__ so that their loads stay behind the
// griddepcontrol.wait (a preceding kernel may have written them).
// kPlan: one more block computes the length-aware plan (batch > 1).
// kRows: 0 = every absorb block takes all rows; 1 = kAbsorbRows query rows each
// (kAbsorbBlocks blocks per kAbsorbRows rows); 2 = the rope columns only, kRopeRows
// rows of all heads per block (a prompt chunk, whose latent part the tensor-core
// absorb computes).
// Mode 2 blocks take kRopeRows rows of all 32 heads each (q_rope_rows_block).
constexpr int kRopeRows = 4;

// The block-table lines of WorkPlanArgs, shared out over every thread of the
// grid.  The table is not written by this kernel or the preceding one in a
// decode call, and a prefetch only moves a line into L2, so it is issued at
// once, before any wait.
__device__ __forceinline__ void prefetch_block_table(const WorkPlanArgs& a) {
  const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
  for (int64_t l = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; l < a.bt_lines; l += nthr)
    prefetch_l2(a.bt_prefetch + l * 32);
}

template <int kRows>
struct AbsorbGrid {
  static constexpr int kPerRows = kRows == 2 ? kHeads : kAbsorbBlocks;
  __host__ __device__ __forceinline__ static int blocks(int rows) {
    if constexpr (kRows == 2) return (rows + kRopeRows - 1) / kRopeRows;
    return kRows ? kPerRows * ((rows + kAbsorbRows - 1) / kAbsorbRows) : kAbsorbBlocks;
  }
  // block -> (head, column block, first row, end row)
  __device__ __forceinline__ static void map(int blk, int rows, int& h, int& cb, int& r_lo,
                                             int& r_hi) {
    const int hb = kRows ? blk % kPerRows : blk;
    r_lo = kRows ? (blk / kPerRows) * kAbsorbRows : 0;
    r_hi = kRows ? min(rows, r_lo + kAbsorbRows) : rows;
    h = kRows == 2 ? hb : hb % kHeads;
    cb = kRows == 2 ? kDLatent / 64 : hb / kHeads;
  }
};

template <bool kPlan, int kRows, bool kF16 = false>
__global__ void __launch_bounds__(kAbsorbThreads) q_absorb_kernel(
    const __nv_bfloat16* q, const __nv_bfloat16* __restrict__ W_UK, const int32_t* seqlens,
    __nv_bfloat16* __restrict__ q_ext, int rows, int q_len, int split, float qscale,
    const RopeTable tab, const WorkPlanArgs plan) {
  __shared__ union {
    AbsorbSmem absorb;
    PlanSmem plan;
  } sm;
  // every role signals dependent launches right after its own wait for the
  // preceding kernel: a dependent grid starts only once every kernel older than
  // this one has completed (the split-K kernel reads sequence lengths and block
  // ids before its own wait, relying on that)
  prefetch_block_table(plan);
  using G = AbsorbGrid<kRows>;
  const int absorb_blocks = G::blocks(rows);
  if constexpr (kPlan) {
    if (blockIdx.x == absorb_blocks) {
      work_plan_block(plan, sm.plan);
      return;
    }
  }
  if constexpr (kRows == 2) {
    const int r_lo = blockIdx.x * kRopeRows;
    q_rope_rows_block(r_lo, min(rows, r_lo + kRopeRows), q, seqlens, q_ext, q_len, split, qscale,
                      tab, sm.absorb);
    return;
  }
  int h, cb, r_lo, r_hi;
  G::map(blockIdx.x, rows, h, cb, r_lo, r_hi);
  q_absorb_block<kRows != 0, kF16>(h, cb, q, W_UK, seqlens, q_ext, rows, q_len, split, qscale,
                                   tab, sm.absorb, r_lo, r_hi);
}

// The first kernel of a decode step: the absorb blocks above, then the
// producer's blocks when the step starts from hidden states (produce.cuh, 4
// warps each; pa.T == 0 otherwise), then blocks that append the step's ready
// cache rows (one thread per 16-byte piece).  All of them only wait for the
// kernel launched before this one, so they run side by side.
// kPlan: one more block computes the length-aware plan (batch > 1); the
// producer and append blocks follow it.  kRows as for q_absorb_kernel.
template <bool kPlan, int kRows>
__global__ void __launch_bounds__(kAbsorbThreads) step_prologue_kernel(
    const __nv_bfloat16* q, const __nv_bfloat16* __restrict__ W_UK, const int32_t* seqlens,
    __nv_bfloat16* __restrict__ q_ext, int rows, int q_len, int split, float qscale,
    const RopeTable q_tab, const AppendArgs ap, const RopeTable k_tab, const ProduceArgs pa,
    const WorkPlanArgs plan) {
  // one buffer for whichever role the block takes
  __shared__ union {
    AbsorbSmem absorb;
    ProduceSmem<kAbsorbThreads / 32> produce;
    PlanSmem plan;
  } sm;
  // every role signals dependent launches right after its own wait (as in
  // q_absorb_kernel)
  prefetch_block_table(plan);
  using G = AbsorbGrid<kRows>;
  const int absorb_blocks = G::blocks(rows);
  if (blockIdx.x < absorb_blocks) {
    if constexpr (kRows == 2) {
      const int r_lo = blockIdx.x * kRopeRows;
      q_rope_rows_block(r_lo, min(rows, r_lo + kRopeRows), q, seqlens, q_ext, q_len, split,
                        qscale, q_tab, sm.absorb);
      return;
    }
    int h, cb, r_lo, r_hi;
    G::map(blockIdx.x, rows, h, cb, r_lo, r_hi);
    q_absorb_block<kRows != 0>(h, cb, q, W_UK, seqlens, q_ext, rows, q_len, split, qscale, q_tab,
                               sm.absorb, r_lo, r_hi);
    return;
  }
  constexpr int kPlanBlocks = kPlan ? 1 : 0;
  if constexpr (kPlan) {
    if (blockIdx.x == absorb_blocks) {
      work_plan_block(plan, sm.plan);
      return;
    }
  }
  const int prod_blocks = pa.T > 0 ? kProdBlocks : 0;
  if (blockIdx.x < absorb_blocks + kPlanBlocks + prod_blocks) {
    produce_block<kAbsorbThreads / 32>(blockIdx.x - absorb_blocks - kPlanBlocks, threadIdx.x, pa,
                                       k_tab, sm.produce, [] { __syncthreads(); }, [] {
                                         pdl_wait();
                                         pdl_launch_dependents();
                                       });
    return;
  }
  pdl_wait();
  pdl_launch_dependents();
  const int64_t total = ap.T * kRowPieces;
  const int64_t idx =
      (int64_t)(blockIdx.x - absorb_blocks - kPlanBlocks - prod_blocks) * kAbsorbThreads +
      threadIdx.x;
  if (idx < total)
    append_piece(idx, ap.pool, ap.num_blocks, ap.block_table, ap.max_blocks, ap.batch, ap.seq_ids,
                 ap.positions, ap.c_kv, ap.k_pe, ap.status, ap.rotate, k_tab);
}

cudaError_t launch_q_absorb(const __nv_bfloat16* q, const __nv_bfloat16* W_UK,
                            const int32_t* seqlens, __nv_bfloat16* q_ext, int rows, int q_len,
                            int split, float qscale, const RopeTable& tab,
                            const WorkPlanArgs& plan, bool with_plan, bool rope_only,
                            cudaStream_t st, bool f16) {
  const int mode = rope_only ? 2 : rows > kAbsorbRows ? 1 : 0;
  const int64_t nrb = (rows + kAbsorbRows - 1) / kAbsorbRows;
  const unsigned absorb_blocks =
      (unsigned)(mode == 2 ? AbsorbGrid<2>::blocks(rows)
                           : mode == 1 ? kAbsorbBlocks * nrb : kAbsorbBlocks);
  if (with_plan && !plan_ok(plan)) return cudaErrorInvalidValue;
  const unsigned blocks = absorb_blocks + (with_plan ? 1u : 0u);
  if (f16) {
    if (mode == 2) return cudaErrorInvalidValue;
    if (with_plan)
      return launch_pdl(mode == 1 ? q_absorb_kernel<true, 1, true> : q_absorb_kernel<true, 0, true>,
                        dim3(blocks), dim3(kAbsorbThreads), 0, st, q, W_UK, seqlens, q_ext, rows,
                        q_len, 0, qscale, tab, plan);
    return launch_pdl(mode == 1 ? q_absorb_kernel<false, 1, true> : q_absorb_kernel<false, 0, true>,
                      dim3(blocks), dim3(kAbsorbThreads), 0, st, q, W_UK, seqlens, q_ext, rows,
                      q_len, 0, qscale, tab, plan);
  }
  auto kern = [&](bool p) {
    if (p)
      return mode == 2 ? q_absorb_kernel<true, 2> : mode == 1 ? q_absorb_kernel<true, 1>
                                                              : q_absorb_kernel<true, 0>;
    return mode == 2 ? q_absorb_kernel<false, 2> : mode == 1 ? q_absorb_kernel<false, 1>
                                                             : q_absorb_kernel<false, 0>;
  };
  return launch_pdl(kern(with_plan), dim3(blocks), dim3(kAbsorbThreads), 0, st, q, W_UK, seqlens,
                    q_ext, rows, q_len, split, qscale, tab, plan);
}

cudaError_t launch_step_prologue(const __nv_bfloat16* q, const __nv_bfloat16* W_UK,
                                 const int32_t* seqlens, __nv_bfloat16* q_ext, int rows,
                                 int q_len, int split, float qscale, const RopeTable& q_tab,
                                 const AppendArgs& ap, const RopeTable& k_tab,
                                 const ProduceArgs* pa, const WorkPlanArgs& plan, bool with_plan,
                                 bool rope_only, cudaStream_t st) {
  const int64_t append_blocks = (ap.T * kRowPieces + kAbsorbThreads - 1) / kAbsorbThreads;
  if (append_blocks > (1 << 20)) return cudaErrorInvalidValue;
  ProduceArgs none{};
  const ProduceArgs& p = pa != nullptr ? *pa : none;
  const int64_t prod_blocks = p.T > 0 ? kProdBlocks : 0;
  const int mode = rope_only ? 2 : rows > kAbsorbRows ? 1 : 0;
  const int64_t nrb = (rows + kAbsorbRows - 1) / kAbsorbRows;
  const int64_t absorb_blocks = mode == 2   ? (int64_t)AbsorbGrid<2>::blocks(rows)
                               : mode == 1 ? (int64_t)kAbsorbBlocks * nrb
                                           : kAbsorbBlocks;
  auto kern = [&](bool with) {
    if (with)
      return mode == 2 ? step_prologue_kernel<true, 2>
                       : mode == 1 ? step_prologue_kernel<true, 1> : step_prologue_kernel<true, 0>;
    return mode == 2 ? step_prologue_kernel<false, 2>
                     : mode == 1 ? step_prologue_kernel<false, 1> : step_prologue_kernel<false, 0>;
  };
  if (with_plan && !plan_ok(plan)) return cudaErrorInvalidValue;
  const int64_t blocks = absorb_blocks + (with_plan ? 1 : 0) + prod_blocks + append_blocks;
  return launch_pdl(kern(with_plan), dim3((unsigned)blocks), dim3(kAbsorbThreads), 0, st, q, W_UK,
                    seqlens, q_ext, rows, q_len, split, qscale, q_tab, ap, k_tab, p, plan);
}

// ---------------------------------------------------------------- combine + W_UV

// Cluster of 8 CTAs per (head h, chunk of up to kCombineRows output rows).
// CTA `slice` owns latent dims [64 slice, 64 slice + 64).
//  * Merge.  16 groups of 16 threads (one float4 of the slice each) are shared
//    out over the chunk's rows, and a row's splits are dealt round-robin over
//    its groups, so one pass of loads covers the chunk.  Lane k of a group also
//    loads (m, l) of the group's k-th split; a group merges its splits against
//    its own maximum m_g (weights 2^(m_s - m_g), shared by shuffles), so no
//    pass over the row's statistics precedes the loads.  The groups of a row
//    are then combined with weights 2^(m_g - M) against the row maximum M and
//    divided by L = sum_g l_g 2^(m_g - M).  A split that saw no token (l = 0,
//    partial O never written) is skipped, not multiplied by zero.
//  * W_UV.  The merged, normalised 64 dims are multiplied by the slice's 64
//    rows of W_UV[h]; with fewer than 4 rows the 64 dims are also split over
//    the threads.  Each 16-column block of the product is written into the
//    shared memory of the CTA that owns the block (distributed shared memory);
//    the owner adds the 8 contributions in a fixed order and writes out.
constexpr int kSlices = 8;
constexpr int kSliceDims = kDLatent / kSlices;        // 64
constexpr int kCombineRows = 16;
constexpr int kCombineThreads = 256;
constexpr int kCombineGroups = kCombineThreads / 16;  // 16 threads x float4 cover a split row's slice
constexpr int kCombineDepth = 10;                     // split rows each thread keeps in flight (<= 16)
constexpr int kColsPerSlice = kDV / kSlices;          // 16
static_assert(kCombineDepth <= 16, "a group's lanes carry (m, l) of at most 16 splits");

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void fma4(float4& acc, float w, const float4& x) {
  acc.x = fmaf(w, x.x, acc.x);
  acc.y = fmaf(w, x.y, acc.y);
  acc.z = fmaf(w, x.z, acc.z);
  acc.w = fmaf(w, x.w, acc.w);
}

// The merge of one group's splits (sub, sub + gpr, ...) of a row, for the
// float4 q4 of a 64-dim slice: the first kCombineDepth split rows are loaded
// together and merged against the group's maximum over its first 16 splits
// (lane k of the 16-lane group loads (m, l) of the group's k-th split); later
// splits are loaded one by one and merged online.  Splits with l = 0 (no
// token) are skipped.  po / pml: the row's O slice and (m, l) of split 0;
// splits are o_stride floats and ml_stride (m, l) pairs apart.
__device__ __forceinline__ void merge_group(const float* po, const float2* pml, int64_t o_stride,
                                            int64_t ml_stride, int nsplit, int sub, int gpr, int q4,
                                            bool active, float& m_g, float& l_g, float4& acc) {
  float4 v[kCombineDepth];
#pragma unroll
  for (int k = 0; k < kCombineDepth; ++k) {
    const int s = sub + gpr * k;
    v[k] = active && s < nsplit ? *reinterpret_cast<const float4*>(po + s * o_stride)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int s_lane = sub + gpr * q4;  // the split whose (m, l) this lane loads
  const float2 ml = active && s_lane < nsplit ? pml[(int64_t)s_lane * ml_stride]
                                              : make_float2(-INFINITY, 0.f);

  // group maximum over its first 16 splits (lanes of one group: 16 consecutive)
  m_g = ml.y > 0.f ? ml.x : -INFINITY;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m_g = fmaxf(m_g, __shfl_xor_sync(0xffffffffu, m_g, o));
  l_g = 0.f;
  acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kCombineDepth; ++k) {
    const float mk = __shfl_sync(0xffffffffu, ml.x, k, 16);
    const float lk = __shfl_sync(0xffffffffu, ml.y, k, 16);
    if (lk > 0.f) {  // also false past the group's last split
      const float w = ex2(mk - m_g);
      l_g = fmaf(w, lk, l_g);
      fma4(acc, w, v[k]);
    }
  }
  // splits past the first kCombineDepth of the group (many splits per group only):
  // loaded one by one, merged online
  if (active) {
    for (int s = sub + gpr * kCombineDepth; s < nsplit; s += gpr) {
      const float2 x = pml[(int64_t)s * ml_stride];
      if (x.y > 0.f) {
        if (x.x > m_g) {
          const float c = m_g == -INFINITY ? 0.f : ex2(m_g - x.x);
          l_g *= c;
          acc.x *= c;
          acc.y *= c;
          acc.z *= c;
          acc.w *= c;
          m_g = x.x;
        }
        const float w = ex2(x.x - m_g);
        l_g = fmaf(w, x.y, l_g);
        fma4(acc, w, *reinterpret_cast<const float4*>(po + s * o_stride));
      }
    }
  }
}

// kStrided: splits are o_stride floats / ml_stride (m, l) pairs apart (the
// gathered partials of a sequence-parallel decode); otherwise rows_per_cta
// rows apart, as the split-K kernel writes them.  kTable: the splits of a
// (sequence, row group) unit are those unit_tab gives (length-aware plan),
// read after the wait; otherwise nsplit per unit, unit after unit.
// kMinBlocks: CTAs per SM the kernel is compiled for: 3, or 4 when there are
// more than kCombineRows rows, so that 512 CTAs (32 rows) still run in one wave.
template <bool kStrided, bool kTable, int kMinBlocks>
__global__ void __cluster_dims__(kSlices, 1, 1) __launch_bounds__(kCombineThreads, kMinBlocks)
    combine_uv_kernel(const float* part_o, const float* part_ml,
                      const __nv_bfloat16* __restrict__ W_UV, __nv_bfloat16* __restrict__ out,
                      int rows, int q_len, int groups, int nsplit, int rows_per_cta,
                      int64_t o_stride_arg, int64_t ml_stride_arg, const int2* unit_tab) {
  // part_o and part_ml are written by the kernel launched just before this one,
  // which lets this grid start early: they carry no __restrict__, so their loads
  // are not taken as invariant and stay behind the griddepcontrol.wait below.
  __shared__ __align__(16) __nv_bfloat16 w_s[kSliceDims][kDV];  // this slice's rows of W_UV[h]
  __shared__ __align__(16) float4 acc_s[kCombineGroups][kSliceDims / 4];
  __shared__ float grp_m[kCombineGroups], grp_l[kCombineGroups];
  __shared__ __align__(16) float o_s[kCombineRows][kSliceDims];
  __shared__ __align__(16) float prod_s[kCombineRows][kDV];  // [c part * nr + row][v]
  __shared__ __align__(16) float inbox[kSlices][kCombineRows][kColsPerSlice];  // by sender slice
  cg::cluster_group cluster = cg::this_cluster();
  const int slice = (int)cluster.block_rank();
  const int cid = blockIdx.x / kSlices;
  const int h = cid % kHeads;
  const int chunk = cid / kHeads;
  const int r0 = chunk * kCombineRows;
  const int nr = min(kCombineRows, rows - r0);
  const int tid = threadIdx.x;
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

  // thread -> (row, group of the row, float4 of the slice)
  const int q4 = tid & 15;
  const int grp = tid >> 4;
  const int gpr = max(1, kCombineGroups / nr);  // groups per row
  const int my_rr = grp / gpr;
  const int sub = grp % gpr;
  const bool active = my_rr < nr;
  int64_t base = 0;  // partial row of split 0; split s is s * rows_per_cta rows further
  int unit = 0, ridx = 0;
  if (active) {
    const int r = r0 + my_rr;  // r = b*q_len + j
    const int b = r / q_len, j = r % q_len;
    ridx = j * kHeads + h;
    unit = b * groups + ridx / rows_per_cta;
    base = (int64_t)unit * nsplit * rows_per_cta + ridx % rows_per_cta;
  }
  const float* po = part_o + base * kDLatent + slice * kSliceDims + 4 * q4;
  const float2* pml = reinterpret_cast<const float2*>(part_ml) + base;
  const int64_t o_stride = kStrided ? o_stride_arg : rows_per_cta * kDLatent;
  const int64_t ml_stride = kStrided ? ml_stride_arg : rows_per_cta;

  pdl_wait();  // the split partials come from the decode kernel

  int ns = nsplit;
  if constexpr (kTable) {
    // the plan was written by the first kernel of the call, complete before the decode kernel
    const int2 ut = active ? unit_tab[unit] : make_int2(0, 0);
    ns = ut.y;
    base = (int64_t)ut.x * rows_per_cta + ridx % rows_per_cta;
    po = part_o + base * kDLatent + slice * kSliceDims + 4 * q4;
    pml = reinterpret_cast<const float2*>(part_ml) + base;
  }
  float m_g, l_g;
  float4 acc;
  merge_group(po, pml, o_stride, ml_stride, ns, sub, gpr, q4, active, m_g, l_g, acc);
  acc_s[grp][q4] = acc;
  if (q4 == 0) {
    grp_m[grp] = m_g;
    grp_l[grp] = l_g;
  }
  __syncthreads();
  for (int e = tid; e < nr * kSliceDims; e += kCombineThreads) {
    const int rr = e / kSliceDims, d = e % kSliceDims;
    const int g0 = rr * gpr;
    float M = -INFINITY;
    for (int g = 0; g < gpr; ++g) M = fmaxf(M, grp_m[g0 + g]);
    float L = 0.f, t = 0.f;
    for (int g = 0; g < gpr; ++g) {
      if (grp_l[g0 + g] > 0.f) {
        const float w = ex2(grp_m[g0 + g] - M);
        L = fmaf(w, grp_l[g0 + g], L);
        t = fmaf(w, reinterpret_cast<const float*>(&acc_s[g0 + g][0])[d], t);
      }
    }
    o_s[rr][d] = L > 0.f ? t / L : 0.f;
  }
  __syncthreads();

  // slice product prod[r][v] = sum over the slice's 64 dims c of o[r][c] W_UV[h][c][v]:
  // thread = (column pair vp, unit u of 4); with cs = 4 / nr parts of the 64 dims
  // (cs = 1 from 4 rows up), unit u takes dims part u % cs of rows u / cs, u / cs + 4 / cs, ...
  {
    const int vp = tid & (kDV / 2 - 1);
    const int u = tid / (kDV / 2);
    const int cs = nr >= 4 ? 1 : (nr == 1 ? 4 : 2);
    const int cq = u % cs;
    const int c0 = cq * (kSliceDims / cs), c1 = c0 + kSliceDims / cs;
    for (int rr = u / cs; rr < nr; rr += 4 / cs) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 16
      for (int c = c0; c < c1; ++c) {
        const float2 w = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(&w_s[c][0])[vp]);
        const float x = o_s[rr][c];
        a0 = fmaf(x, w.x, a0);
        a1 = fmaf(x, w.y, a1);
      }
      *reinterpret_cast<float2*>(&prod_s[cq * nr + rr][2 * vp]) = make_float2(a0, a1);
    }
    __syncthreads();
    cluster_wait_acquire();  // every CTA of the cluster is running
    for (int e = tid; e < nr * kDV; e += kCombineThreads) {
      const int rr = e / kDV, v = e % kDV;
      float t = prod_s[rr][v];
      for (int k = 1; k < cs; ++k) t += prod_s[k * nr + rr][v];
      float* dst = cluster.map_shared_rank(&inbox[slice][0][0], v / kColsPerSlice);
      dst[rr * kColsPerSlice + v % kColsPerSlice] = t;
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

cudaError_t launch_combine(const float* part_o, const float* part_ml, const __nv_bfloat16* W_UV,
                           __nv_bfloat16* out, int rows, int q_len, int groups, int nsplit,
                           int rows_per_cta, cudaStream_t st, int64_t o_stride,
                           int64_t ml_stride, const int2* unit_tab) {
  const int chunks = (rows + kCombineRows - 1) / kCombineRows;
  const dim3 grid(kSlices * kHeads * chunks);
  const bool strided = o_stride != 0 || ml_stride != 0;
  if (strided && unit_tab != nullptr) return cudaErrorInvalidValue;
  const bool wide = rows > kCombineRows;
  if (unit_tab != nullptr)
    return launch_pdl(wide ? combine_uv_kernel<false, true, 4> : combine_uv_kernel<false, true, 3>,
                      grid, dim3(kCombineThreads), 0, st, part_o, part_ml, W_UV, out, rows, q_len,
                      groups, nsplit, rows_per_cta, (int64_t)0, (int64_t)0, unit_tab);
  if (!strided)
    return launch_pdl(wide ? combine_uv_kernel<false, false, 4> : combine_uv_kernel<false, false, 3>,
                      grid, dim3(kCombineThreads), 0, st, part_o, part_ml, W_UV, out, rows, q_len,
                      groups, nsplit, rows_per_cta, (int64_t)0, (int64_t)0, unit_tab);
  return launch_pdl(wide ? combine_uv_kernel<true, false, 4> : combine_uv_kernel<true, false, 3>,
                    grid, dim3(kCombineThreads), 0, st, part_o, part_ml, W_UV, out, rows, q_len,
                    groups, nsplit, rows_per_cta, o_stride, ml_stride, unit_tab);
}

// ---------------------------------------------------------------- merge of one shard's splits

// One rank's share of a sequence-parallel decode: its splits are merged into
// one partial per (query row, head) -- the running maximum M, the sum L and
// the unnormalised O, all relative to M -- laid out as
//   out[(r * 32 + h) * 512 + d]             O,  r = b * q_len + j
//   out[R * 512 + (r * 32 + h) * 2 + {0,1}] M, L  (R = rows * 32)
// so that the partials of G ranks, gathered one after another, are G splits
// of the combine above (split stride R * 514 floats).  Blocks as in the
// combine: (64-dim slice, head, chunk of up to 16 rows), 256 threads.
__global__ void __launch_bounds__(kCombineThreads)
    merge_splits_kernel(const float* part_o, const float* part_ml, float* __restrict__ out,
                        int rows, int q_len, int groups, int nsplit, int rows_per_cta) {
  __shared__ __align__(16) float4 acc_s[kCombineGroups][kSliceDims / 4];
  __shared__ float grp_m[kCombineGroups], grp_l[kCombineGroups];
  const int slice = blockIdx.x % kSlices;
  const int cid = blockIdx.x / kSlices;
  const int h = cid % kHeads;
  const int chunk = cid / kHeads;
  const int r0 = chunk * kCombineRows;
  const int nr = min(kCombineRows, rows - r0);
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  const int q4 = tid & 15;
  const int grp = tid >> 4;
  const int gpr = max(1, kCombineGroups / nr);
  const int my_rr = grp / gpr;
  const int sub = grp % gpr;
  const bool active = my_rr < nr;
  int64_t base = 0;
  if (active) {
    const int r = r0 + my_rr;
    const int b = r / q_len, j = r % q_len;
    const int ridx = j * kHeads + h;
    base = ((int64_t)b * groups + ridx / rows_per_cta) * nsplit * rows_per_cta + ridx % rows_per_cta;
  }
  const float* po = part_o + base * kDLatent + slice * kSliceDims + 4 * q4;
  const float2* pml = reinterpret_cast<const float2*>(part_ml) + base;
  pdl_wait();  // the split partials come from the decode kernel
  float m_g, l_g;
  float4 acc;
  merge_group(po, pml, (int64_t)rows_per_cta * kDLatent, rows_per_cta, nsplit, sub, gpr, q4,
              active, m_g, l_g, acc);
  acc_s[grp][q4] = acc;
  if (q4 == 0) {
    grp_m[grp] = m_g;
    grp_l[grp] = l_g;
  }
  __syncthreads();
  const int64_t R = (int64_t)rows * kHeads;
  for (int e = tid; e < nr * kSliceDims; e += kCombineThreads) {
    const int rr = e / kSliceDims, d = e % kSliceDims;
    const int g0 = rr * gpr;
    float M = -INFINITY;
    for (int g = 0; g < gpr; ++g)
      if (grp_l[g0 + g] > 0.f) M = fmaxf(M, grp_m[g0 + g]);
    float L = 0.f, t = 0.f;
    for (int g = 0; g < gpr; ++g) {
      if (grp_l[g0 + g] > 0.f) {
        const float w = ex2(grp_m[g0 + g] - M);
        L = fmaf(w, grp_l[g0 + g], L);
        t = fmaf(w, reinterpret_cast<const float*>(&acc_s[g0 + g][0])[d], t);
      }
    }
    const int64_t row = (int64_t)(r0 + rr) * kHeads + h;
    out[row * kDLatent + slice * kSliceDims + d] = t;
    if (slice == 0 && d == 0) {
      out[R * kDLatent + 2 * row] = M;
      out[R * kDLatent + 2 * row + 1] = L;
    }
  }
}

// ---------------------------------------------------------------- latent output of a prompt chunk

// For the tensor-core W_UV product of a prompt chunk: the splits of each
// (row, head) merged and normalised, o = sum_s 2^(m_s - M) O_s / L, written as
// o_hi = bf16(o) and o_lo = bf16(o - o_hi) at [(r * 32 + h) * 512 + d].  Blocks
// as in the combine (64-dim slice, head, chunk of up to 16 rows), 256 threads.
template <bool kTable>
__global__ void __launch_bounds__(kCombineThreads)
    latent_out_kernel(const float* part_o, const float* part_ml, __nv_bfloat16* __restrict__ o_hi,
                      __nv_bfloat16* __restrict__ o_lo, int rows, int q_len, int groups,
                      int nsplit, int rows_per_cta, const int2* unit_tab) {
  __shared__ __align__(16) float4 acc_s[kCombineGroups][kSliceDims / 4];
  __shared__ float grp_m[kCombineGroups], grp_l[kCombineGroups];
  const int slice = blockIdx.x % kSlices;
  const int cid = blockIdx.x / kSlices;
  const int h = cid % kHeads;
  const int chunk = cid / kHeads;
  const int r0 = chunk * kCombineRows;
  const int nr = min(kCombineRows, rows - r0);
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  const int q4 = tid & 15;
  const int grp = tid >> 4;
  const int gpr = max(1, kCombineGroups / nr);
  const int my_rr = grp / gpr;
  const int sub = grp % gpr;
  const bool active = my_rr < nr;
  int unit = 0, ridx = 0;
  if (active) {
    const int r = r0 + my_rr;
    const int b = r / q_len, j = r % q_len;
    ridx = j * kHeads + h;
    unit = b * groups + ridx / rows_per_cta;
  }
  pdl_wait();  // the split partials come from the decode kernel
  int64_t base = (int64_t)unit * nsplit * rows_per_cta + ridx % rows_per_cta;
  int ns = nsplit;
  if constexpr (kTable) {
    const int2 ut = active ? unit_tab[unit] : make_int2(0, 0);
    ns = ut.y;
    base = (int64_t)ut.x * rows_per_cta + ridx % rows_per_cta;
  }
  const float* po = part_o + base * kDLatent + slice * kSliceDims + 4 * q4;
  const float2* pml = reinterpret_cast<const float2*>(part_ml) + base;
  float m_g, l_g;
  float4 acc;
  merge_group(po, pml, (int64_t)rows_per_cta * kDLatent, rows_per_cta, ns, sub, gpr, q4, active,
              m_g, l_g, acc);
  acc_s[grp][q4] = acc;
  if (q4 == 0) {
    grp_m[grp] = m_g;
    grp_l[grp] = l_g;
  }
  __syncthreads();
  for (int e = tid; e < nr * kSliceDims / 2; e += kCombineThreads) {
    const int rr = e / (kSliceDims / 2), d = 2 * (e % (kSliceDims / 2));
    const int g0 = rr * gpr;
    float M = -INFINITY;
    for (int g = 0; g < gpr; ++g)
      if (grp_l[g0 + g] > 0.f) M = fmaxf(M, grp_m[g0 + g]);
    float L = 0.f, t0 = 0.f, t1 = 0.f;
    for (int g = 0; g < gpr; ++g) {
      if (grp_l[g0 + g] > 0.f) {
        const float w = ex2(grp_m[g0 + g] - M);
        L = fmaf(w, grp_l[g0 + g], L);
        t0 = fmaf(w, reinterpret_cast<const float*>(&acc_s[g0 + g][0])[d], t0);
        t1 = fmaf(w, reinterpret_cast<const float*>(&acc_s[g0 + g][0])[d + 1], t1);
      }
    }
    const float a = L > 0.f ? t0 / L : 0.f, c = L > 0.f ? t1 / L : 0.f;
    const __nv_bfloat162 hv = __floats2bfloat162_rn(a, c);
    const __nv_bfloat162 lv = __floats2bfloat162_rn(a - __low2float(hv), c - __high2float(hv));
    const int64_t off = ((int64_t)(r0 + rr) * kHeads + h) * kDLatent + slice * kSliceDims + d;
    *reinterpret_cast<__nv_bfloat162*>(o_hi + off) = hv;
    *reinterpret_cast<__nv_bfloat162*>(o_lo + off) = lv;
  }
}

cudaError_t launch_latent_out(const float* part_o, const float* part_ml, __nv_bfloat16* o_hi,
                              __nv_bfloat16* o_lo, int rows, int q_len, int groups, int nsplit,
                              int rows_per_cta, const int2* unit_tab, cudaStream_t st) {
  const int chunks = (rows + kCombineRows - 1) / kCombineRows;
  const dim3 grid(kSlices * kHeads * chunks);
  if (unit_tab != nullptr)
    return launch_pdl(latent_out_kernel<true>, grid, dim3(kCombineThreads), 0, st, part_o, part_ml,
                      o_hi, o_lo, rows, q_len, groups, nsplit, rows_per_cta, unit_tab);
  return launch_pdl(latent_out_kernel<false>, grid, dim3(kCombineThreads), 0, st, part_o, part_ml,
                    o_hi, o_lo, rows, q_len, groups, nsplit, rows_per_cta, unit_tab);
}

cudaError_t launch_merge_splits(const float* part_o, const float* part_ml, float* out, int rows,
                                int q_len, int groups, int nsplit, int rows_per_cta,
                                cudaStream_t st) {
  const int chunks = (rows + kCombineRows - 1) / kCombineRows;
  return launch_pdl(merge_splits_kernel, dim3(kSlices * kHeads * chunks), dim3(kCombineThreads), 0,
                    st, part_o, part_ml, out, rows, q_len, groups, nsplit, rows_per_cta);
}

}  // namespace xmla
