// One 16-byte piece of a paged-cache append.
//
// [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section "MLA：256K 上下文的
//      '内存革命'": the cache row of a token is its 512-dim latent c_kv followed by
//      its 64-dim rope key.  Shared by the standalone append kernel and the fused
//      prologue of a decode step.
#pragma once

#include <cstdint>

#include "xmla_device.cuh"
#include "yarn.cuh"

namespace xmla {

constexpr int kLatPieces = kDLatent * 2 / 16;  // 64 pieces of latent per row
constexpr int kRopePieces = kDRope * 2 / 16;   // 8 pieces of rope key per row
constexpr int kRowPieces = kLatPieces + kRopePieces;

// Piece `idx` (row t = idx / 72, piece idx % 72) of the rows being appended:
// latent pieces are bit copies; rope pieces are bit copies too unless `rotate`,
// in which case rope piece r rotates the four pairs (4r .. 4r+3, 4r+32 .. 4r+35)
// at the row's position (angle in float64, one rounding to bf16).  A row whose
// sequence, position or block id is out of range is skipped and
// XMLA_ERR_DEVICE_OOB recorded.  No pointer argument is __restrict__: the
// kernel launched just before may have written them (see griddepcontrol.wait).
__device__ __forceinline__ void append_piece(int64_t idx, uint4* pool, int64_t num_blocks,
                                             const int32_t* block_table, int32_t max_blocks,
                                             int32_t batch, const int32_t* seq_ids,
                                             const int64_t* positions, const uint4* c_kv,
                                             const uint4* k_pe, int32_t* status, int rotate,
                                             const RopeTable& tab) {
  const int64_t t = idx / kRowPieces;
  const int piece = (int)(idx % kRowPieces);
  const int32_t s = seq_ids[t];
  const int64_t pos = positions[t];
  if (s < 0 || s >= batch || pos < 0 || pos >= (int64_t)max_blocks * kPage) {
    record_status(status, XMLA_ERR_DEVICE_OOB);
    return;
  }
  const int32_t blk = block_table[(int64_t)s * max_blocks + pos / kPage];
  if (blk < 0 || (int64_t)blk >= num_blocks) {
    record_status(status, XMLA_ERR_DEVICE_OOB);
    return;
  }
  uint4* row = pool + ((int64_t)blk * kPage + pos % kPage) * kRowPieces;
  if (piece < kLatPieces) {
    row[piece] = c_kv[t * kLatPieces + piece];
  } else if (!rotate) {
    row[piece] = k_pe[t * kRopePieces + (piece - kLatPieces)];
  } else {
    const int r = piece - kLatPieces;  // pairs 4r .. 4r+3
    const uint2* src = reinterpret_cast<const uint2*>(k_pe + t * kRopePieces);
    uint2* dst = reinterpret_cast<uint2*>(row + kLatPieces);
    const uint2 lo = src[r], hi = src[r + 8];  // dims 4r.., 32+4r..
    const __nv_bfloat16* xl = reinterpret_cast<const __nv_bfloat16*>(&lo);
    const __nv_bfloat16* xh = reinterpret_cast<const __nv_bfloat16*>(&hi);
    uint2 olo, ohi;
    __nv_bfloat16* yl = reinterpret_cast<__nv_bfloat16*>(&olo);
    __nv_bfloat16* yh = reinterpret_cast<__nv_bfloat16*>(&ohi);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      double y1, y2;
      rope_pair((double)__bfloat162float(xl[e]), (double)__bfloat162float(xh[e]), pos, 4 * r + e,
                tab, &y1, &y2);
      yl[e] = __double2bfloat16(y1);
      yh[e] = __double2bfloat16(y2);
    }
    dst[r] = olo;
    dst[r + 8] = ohi;
  }
}

}  // namespace xmla
