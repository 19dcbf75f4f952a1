// One warp's share of the dual-domain attention of a block of 8 clips of one
// (position, head), on tiles staged in shared memory by TMA.  Shared by the
// attention kernel and the attention kernel with the fused output projection.
//
// Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
// write-up), attention-module paragraph: every query frame of clip i attends
// over the clip's own L frames, the last n_pre frames of clip i-1 and the
// first n_post frames of clip i+1 (absent at the video ends) and n_global
// frames sampled over the whole video; duplicates kept, scale 1/sqrt(d).
#pragma once

#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

constexpr int FA_CLIPS = 8;                       // clips per CTA (one per warp)
constexpr int FA_L = 16;                          // frames per clip
constexpr int FA_HALO = 8;                        // halo rows of a shard's padded k/v storage
constexpr int FA_HALO_MAX = 16;                   // max n_pre / n_post of the fast path (= L)
constexpr int FA_NG = 16;                         // max n_global
constexpr int FA_ROWS_Q = FA_CLIPS * FA_L;        // 128 query rows
constexpr int FA_ROW_BYTES = 128;                 // 64 bf16 channels of one head

// Shared-memory layout of the kernel for halo width H (8: every n_pre,
// n_post <= 8; 16: up to a whole clip): Q | K window | V window | K global |
// V global | barrier, the swizzled regions on 1024-byte boundaries.
template <int H>
struct FaLayout {
  static constexpr int ROWS_W = FA_ROWS_Q + 2 * H;      // 144 or 160 window rows
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_KW = OFF_Q + FA_ROWS_Q * FA_ROW_BYTES;
  static constexpr uint32_t OFF_VW = OFF_KW + ROWS_W * FA_ROW_BYTES;
  static constexpr uint32_t OFF_KG = OFF_VW + ROWS_W * FA_ROW_BYTES;
  static constexpr uint32_t OFF_VG = OFF_KG + FA_NG * FA_ROW_BYTES;
  static constexpr uint32_t STAGE = OFF_VG + FA_NG * FA_ROW_BYTES;   // Q .. V global
  static constexpr uint32_t OFF_BAR = STAGE;
  static constexpr uint32_t SMEM = OFF_BAR + 16 + 1024;   // + slack for 1024B alignment
  static_assert(OFF_KW % 1024 == 0 && OFF_VW % 1024 == 0 && OFF_KG % 1024 == 0 &&
                    OFF_VG % 1024 == 0,
                "128B-swizzled regions must start on 1024-byte boundaries");
  static_assert(STAGE % 1024 == 0, "stages stack on 1024-byte boundaries");
};

// Byte address of 16-byte chunk `chunk` of row `row` in a 128B-swizzled region.
__device__ __forceinline__ uint32_t sw128(uint32_t region, int row, int chunk) {
  return region + row * FA_ROW_BYTES + (((chunk ^ (row & 7)) & 7) << 4);
}

// Warp `warp` of the block computes the 16 query rows 16*warp .. 16*warp+15
// of the Q tile against the 2H + 16 window rows 16*warp .. 16*warp + 2H + 15
// and the 16 global keys, and writes its 16 rows of O (bf16, normalised) over
// the same rows of the Q tile, in the tile's 128-byte swizzle.
//   LQ = 16 (clips of 16 frames): the rows are clip `gclip` (its index in the
//   whole video of n_total clips), its window keys C_pre | own | C_post.
//   LQ = 32 (H = 8): the rows are half of clip `gclip`, whose 48 window keys
//   start at window row 32 * (warp / 2).
//   LQ = 8 (clips of 8 frames, H = 8): rows 0-7 are clip gclip and rows 8-15
//   clip gclip + 1; their windows (8 | 8 | 8 keys) are window rows 0-23 and
//   8-31 of the warp's 32.  In the mma.sync accumulator layout a thread holds
//   rows g and g + 8, one of each clip, so each takes its own clip's mask.
//   S = Q K^T and O = P V on tensor cores (mma.sync m16n8k16, bf16 in, fp32
//   accumulate), the softmax in fp32 registers with quad shuffles in log2
//   units (scale_log2 = log2(e)/sqrt(d)); P is rounded to bf16 for the P V
//   product and the row sums use the rounded values.  Keys outside the clip's
//   list (absent ends, n_pre / n_post below H, n_global below 16) are masked
//   to -inf.  Without global frames their tiles are not read at all.
template <int H, int LQ = FA_L>
__device__ __forceinline__ void fa_attend_warp(uint32_t sQ, uint32_t sKW, uint32_t sVW,
                                               uint32_t sKG, uint32_t sVG, int warp, int lane,
                                               int gclip, int n_total, int n_pre, int n_post,
                                               int n_global, float scale_log2) {
  // Window keys of the warp: its clip's (L >= 16: H | L | H), or the union
  // of its two clips' (L = 8: 32).
  constexpr int NW = 2 * H + (LQ >= FA_L ? LQ : FA_L);
  constexpr int NTW = NW / 8;             // their n-tiles
  constexpr int NT = NTW + FA_NG / 8;     // all n-tiles, the 16 global keys included
  constexpr int KS = NT / 2;              // k-steps of P.V
  static_assert(LQ == FA_L || ((LQ == 8 || LQ == 32) && H == 8),
                "clips of 16 frames, or of 8 or 32 with H = 8");
  static_assert(NW % 16 == 0, "whole P.V k-steps over the window");
  // First window row of the warp's keys: its clip's first pre row (L >= 16:
  // warps 2m and 2m+1 share the clip of L = 32), or its first clip's (L = 8).
  const int kbase = LQ > FA_L ? (16 * warp / LQ) * LQ : 16 * warp;
  const int g = lane >> 2, qd = lane & 3;
  // ---- S = Q K^T over 2H + 32 keys (NT n-tiles of 8), 4 k-steps of 16 dims ----
  uint32_t qa[4][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    ldsm_x4(sw128(sQ, warp * 16 + (lane & 15), 2 * ks + (lane >> 4)), qa[ks][0], qa[ks][1],
            qa[ks][2], qa[ks][3]);
  // Without global frames their K/V tiles are not loaded: the MMAs that
  // would read them are skipped (their scores are masked below anyway, but
  // stale shared memory must not reach the P.V product as 0 * NaN).
  const bool has_global = n_global > 0;
  float s[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    if (nt >= NTW && !has_global) continue;
    const uint32_t region = nt < NTW ? sKW : sKG;
    const int row = nt < NTW ? kbase + nt * 8 + (lane & 7) : (nt - NTW) * 8 + (lane & 7);
#pragma unroll
    for (int kp = 0; kp < 2; ++kp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sw128(region, row, 4 * kp + (lane >> 3)), b0, b1, b2, b3);
      mma_bf16_16816(s[nt], qa[2 * kp], b0, b1);
      mma_bf16_16816(s[nt], qa[2 * kp + 1], b2, b3);
    }
  }
  // ---- mask absent keys, softmax in log2 units ----
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int kk = nt * 8 + 2 * qd + c;     // key index in the warp's list
      bool v0, v1;                            // for rows g and g + 8
      if (kk >= NW) {
        v0 = v1 = kk - NW < n_global;
      } else if constexpr (LQ >= FA_L) {
        if (kk < H) v0 = gclip > 0 && kk >= H - n_pre;
        else if (kk < H + LQ) v0 = true;
        else v0 = gclip < n_total - 1 && kk - (H + LQ) < n_post;
        v1 = v0;
      } else {
        // clip gclip + hr sees window keys 8hr .. 8hr + 23 as pre | own | post
        // (a clip past the video's last has no rows in the output: its own
        // keys keep its softmax finite)
        bool v[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int gc = gclip + hr, kl = kk - 8 * hr;
          if (kl < 0 || kl >= 24) v[hr] = false;
          else if (kl < 8) v[hr] = gc > 0 && kl >= 8 - n_pre;
          else if (kl < 16) v[hr] = true;
          else v[hr] = gc < n_total - 1 && kl - 16 < n_post;
        }
        v0 = v[0];
        v1 = v[1];
      }
      s[nt][c] = v0 ? s[nt][c] * scale_log2 : -INFINITY;
      s[nt][c + 2] = v1 ? s[nt][c + 2] * scale_log2 : -INFINITY;
      mx0 = fmaxf(mx0, s[nt][c]);
      mx1 = fmaxf(mx1, s[nt][c + 2]);
    }
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  // P in bf16 as mma A fragments: k-step ks covers keys 16ks .. 16ks+15.
  uint32_t pa[KS][4];
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint32_t lo = pack2_bf16(exp2f(s[nt][0] - mx0), exp2f(s[nt][1] - mx0));
    const uint32_t hi = pack2_bf16(exp2f(s[nt][2] - mx1), exp2f(s[nt][3] - mx1));
    l0 += __uint_as_float(lo << 16) + __uint_as_float(lo & 0xFFFF0000u);
    l1 += __uint_as_float(hi << 16) + __uint_as_float(hi & 0xFFFF0000u);
    pa[nt >> 1][(nt & 1) * 2 + 0] = lo;
    pa[nt >> 1][(nt & 1) * 2 + 1] = hi;
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  // ---- O = P V: KS k-steps of 16 keys x 8 n-tiles of 8 dims ----
  float o[8][4];
#pragma unroll
  for (int nd = 0; nd < 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    if (ks == KS - 1 && !has_global) continue;
    const uint32_t region = ks < KS - 1 ? sVW : sVG;
    const int row = (ks < KS - 1 ? kbase + ks * 16 : 0) + (lane & 15);
#pragma unroll
    for (int nd = 0; nd < 8; nd += 2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sw128(region, row, nd + (lane >> 4)), b0, b1, b2, b3);
      mma_bf16_16816(o[nd], pa[ks], b0, b1);
      mma_bf16_16816(o[nd + 1], pa[ks], b2, b3);
    }
  }
  // ---- normalise, round, write this warp's 16 rows into the Q buffer ----
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int r0 = warp * 16 + g, r1 = r0 + 8;
#pragma unroll
  for (int nd = 0; nd < 8; ++nd) {
    const uint32_t w0 = pack2_bf16(o[nd][0] * inv0, o[nd][1] * inv0);
    const uint32_t w1 = pack2_bf16(o[nd][2] * inv1, o[nd][3] * inv1);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(sw128(sQ, r0, nd) + 4 * qd), "r"(w0));
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(sw128(sQ, r1, nd) + 4 * qd), "r"(w1));
  }
}

}  // namespace vi
