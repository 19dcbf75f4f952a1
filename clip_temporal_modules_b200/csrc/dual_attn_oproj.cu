// Dual-domain temporal attention with the attention module's output
// projection fused in (bf16; the attention fast path's shapes, C <= 320).
//
// Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
// write-up), attention-module paragraph: the module gathers its keys and
// values from the clip, its neighbours and the global frames; the linear
// layers around the attention are the module's own.  Here
//   out = a W_out^T + b_out,
// a [P][F][C] being the dual-domain attention of q, k, v (heads of d = 64
// channels side by side), W_out [C][C] and b_out [C] in the Linear layout.
//
// The attention kernel followed by the output GEMM writes a to HBM and reads
// it back: 2 x 2 bytes per channel and token on top of q, k, v and out.  Here
// a never leaves the SM.
//   Work item = (position p, block of 128 frames), every head.  One
//   persistent CTA per SM walks its items; 10 warps:
//     warps 0-7  the attention (warp w: frames 16w .. 16w+15 of the block, one
//                clip of 16 frames, two of 8 or half of one of 32, the same
//                per-warp code as the attention kernel), then the block's
//                epilogue;
//     warp 8     TMA producer: per head, its stage (Q, K/V window, K/V global)
//                into a ring of 3 stages that runs on across blocks, and the
//                columns 64h .. 64h+63 of W_out (C rows x 128 bytes) into one
//                buffer; it also issues the blocks' output stores;
//     warp 9     TMEM allocation and the MMA thread.
//   Per head, the attention warps write O_h (128 x 64 bf16) over the Q tile
//   of its stage.  That tile's 128-byte swizzle is also the K-major operand
//   layout of tcgen05.mma, so the MMA thread accumulates
//     acc += O_h W_out[:, 64h .. 64h+63]^T
//   into TMEM straight from it (128 lanes x C fp32 columns; 2 x 4 MMAs of
//   M = 128, N = C/2, K = 16 per head).  When the MMAs of head g are done,
//   its stage and the W_out buffer are free: the producer loads the W_out
//   slice of head g+1 and the stage of head g+3.
//   After a block's last head the attention warps read the accumulator (warp
//   w: TMEM lanes 32(w%4) .. +31, columns (w/4)C/2 .. +C/2-1), hand TMEM back
//   to the next block's MMAs, add b_out, round to bf16 and stage the rows in
//   the last head's stage and the W_out buffer; the producer stores them with
//   TMA (frames past the end fall outside the tensor map and are dropped) and
//   refills that memory once the stores have read it.  Meanwhile the
//   attention warps go on with the next block, whose first two stages are
//   already loaded.
// HBM traffic per token: q, k, v read once and out written once (4 C x 2 B),
// against 6 C x 2 B for the attention plus the output GEMM.  Every block
// re-reads W_out (C x C x 2 B) from L2.
#include <atomic>

#include "dual_attn_tile.cuh"
#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

constexpr int FO_THREADS = 320;                   // 8 attention warps, producer, MMA
constexpr int FO_C_MAX = 320;                     // channels (5 heads of 64)
constexpr int FO_STAGES = 3;
constexpr int FO_G_MAX = FO_C_MAX / 64;           // 32-column groups per epilogue warp

// Shared memory: 3 stages of the attention kernel's layout (without its
// barrier) | W_out slice of one head (up to FO_C_MAX rows x 128 B) | barriers.
// The output staging of a block (C/64 boxes of 128 frames x 64 channels,
// 16 KB each) reuses the stage of its last head (boxes 0-2) and the W_out
// buffer (boxes 3-4), both idle from the last head's MMAs until the stores
// have read them.
template <int H>
struct FoLayout {
  static constexpr uint32_t STAGE = FaLayout<H>::STAGE;
  static constexpr uint32_t OFF_W = FO_STAGES * STAGE;
  static constexpr uint32_t OFF_BAR = OFF_W + FO_C_MAX * FA_ROW_BYTES;
  static constexpr uint32_t BOX = FA_ROWS_Q * FA_ROW_BYTES;     // one output box
  static constexpr int BOXES_IN_STAGE = STAGE / BOX;            // 3
  // full[3], o_full[3], w_full, m_done, acc_full, tmem_empty, staged, drain
  // (8 bytes each), TMEM slot; then b_out in fp32
  static constexpr uint32_t OFF_BIAS = OFF_BAR + 128;
  static constexpr uint32_t SMEM = OFF_BIAS + FO_C_MAX * 4 + 1024;   // + slack for alignment
  static_assert(OFF_W % 1024 == 0, "the W_out slice is 128B-swizzled");
  static_assert(BOXES_IN_STAGE >= 3 &&
                    (FO_C_MAX / 64 - BOXES_IN_STAGE) * BOX <= FO_C_MAX * FA_ROW_BYTES,
                "a block's output staging fits one stage and the W_out buffer");
  static_assert(SMEM <= 232448, "one CTA per SM must fit");
};

struct FoMaps {
  CUtensorMap q, k, v, kg, vg;   // as in the attention kernel
  CUtensorMap w;                 // W_out [C][C]: box of 64 input channels x C/2 rows
  CUtensorMap y;                 // out [P][F][C]: box of 64 channels x 128 frames
};

// Persistent: CTA c walks the blocks (position p, 128 frames) c, c + grid,
// ... of the video (N clips of LQ = 8, 16 or 32 frames, P positions); global head
// g of the CTA is head g % heads of its block g / heads, staged in stage g % 3.
// tmem_cols: a power of two >= C.
template <int H, int LQ>
__global__ void __launch_bounds__(FO_THREADS, 1)
    dual_attn_oproj_bf16(const __grid_constant__ FoMaps maps, const bf16* __restrict__ b_out,
                         int N, int P, int heads, int n_pre, int n_post, int n_global,
                         float scale_log2, uint32_t tmem_cols, unsigned int* err_word) {
  using Lay = FaLayout<H>;
  using FL = FoLayout<H>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sW = base + FL::OFF_W, bars = base + FL::OFF_BAR, sBias = base + FL::OFF_BIAS;
  const uint32_t o_full0 = bars + 8 * FO_STAGES, w_full = bars + 16 * FO_STAGES;
  const uint32_t m_done = w_full + 8, acc_full = w_full + 16, tmem_empty = w_full + 24;
  const uint32_t staged = w_full + 32, drain = w_full + 40, tmem_slot = w_full + 48;
  const int C = heads * 64, NH = C / 2;           // NH: N of one MMA, columns of one warp
  const int cpb = FA_ROWS_Q / LQ;                 // clips per block
  const int nblk = (N + cpb - 1) / cpb;
  const long long n_items = (long long)P * nblk;
  const int my_items = (int)((n_items - blockIdx.x + gridDim.x - 1) / gridDim.x);
  const int total = my_items * heads;             // this CTA's heads, all blocks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Block i of this CTA: its position and first frame.
  auto item_pos = [&](int i, int& p, int& f0) {
    const long long it = blockIdx.x + (long long)i * gridDim.x;
    p = (int)(it / nblk);
    f0 = (int)(it % nblk) * FA_ROWS_Q;
  };
  // Output box b of a block staged where its last head's stage and the W_out
  // buffer are.
  auto box_addr = [&](int i, int b) -> uint32_t {
    const int s_last = (i * heads + heads - 1) % FO_STAGES;
    return b < FL::BOXES_IN_STAGE ? base + (uint32_t)s_last * Lay::STAGE + (uint32_t)b * FL::BOX
                                  : sW + (uint32_t)(b - FL::BOXES_IN_STAGE) * FL::BOX;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < FO_STAGES; ++s) {
      mbar_init(bars + 8 * s, 1);
      mbar_init(o_full0 + 8 * s, FA_CLIPS);       // one arrive per attention warp
    }
    mbar_init(w_full, 1);
    mbar_init(m_done, 1);
    mbar_init(acc_full, 1);
    mbar_init(tmem_empty, FA_CLIPS);
    mbar_init(staged, FA_CLIPS);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  if ((int)threadIdx.x < C)                       // C <= FO_C_MAX = FO_THREADS
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(sBias + 4u * threadIdx.x),
                 "f"(__bfloat162float(b_out[threadIdx.x])));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t tmem_base;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem_base) : "r"(tmem_slot));

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t stage_bytes = (FA_ROWS_Q + 2 * Lay::ROWS_W) * FA_ROW_BYTES +
                                   (n_global > 0 ? 2 * FA_NG * FA_ROW_BYTES : 0);
      auto load_stage = [&](int g) {
        int p, f0;
        item_pos(g / heads, p, f0);
        const int h = g % heads;
        const uint32_t st = base + (uint32_t)(g % FO_STAGES) * Lay::STAGE;
        const uint32_t bar = bars + 8 * (g % FO_STAGES);
        mbar_arrive_expect_tx(bar, stage_bytes);
        tma_load_3d(st + Lay::OFF_Q, &maps.q, h * 64, f0, p, bar);
        tma_load_3d(st + Lay::OFF_KW, &maps.k, h * 64, f0 - H, p, bar);
        tma_load_3d(st + Lay::OFF_VW, &maps.v, h * 64, f0 - H, p, bar);
        if (n_global > 0) {
          tma_load_3d(st + Lay::OFF_KG, &maps.kg, h * 64, 0, p, bar);
          tma_load_3d(st + Lay::OFF_VG, &maps.vg, h * 64, 0, p, bar);
        }
      };
      auto load_w = [&](int g) {
        const int h = g % heads;
        mbar_arrive_expect_tx(w_full, (uint32_t)C * FA_ROW_BYTES);
        tma_load_2d(sW, &maps.w, h * 64, 0, w_full);
        tma_load_2d(sW + (uint32_t)NH * FA_ROW_BYTES, &maps.w, h * 64, NH, w_full);
      };
      // Block i's output, once the attention warps have staged it: one TMA
      // store per 64 channels (frames past the end are dropped), the boxes in
      // the W_out buffer first, each region in a bulk group of its own, so
      // that the buffer can be refilled as soon as its boxes have been read.
      const int n_box = C / 64, n_box_w = n_box > FL::BOXES_IN_STAGE ? n_box - FL::BOXES_IN_STAGE : 0;
      auto store_item = [&](int i) -> bool {
        if (!mbar_wait_bounded(staged, (uint32_t)(i & 1), err_word, VI_DEV_ERR_MMA_TIMEOUT))
          return false;
        int p, f0;
        item_pos(i, p, f0);
        for (int b = n_box - n_box_w; b < n_box; ++b)
          tma_store_3d(&maps.y, box_addr(i, b), 64 * b, f0, p);
        bulk_commit();
        for (int b = 0; b < n_box - n_box_w; ++b)
          tma_store_3d(&maps.y, box_addr(i, b), 64 * b, f0, p);
        bulk_commit();
        return true;
      };
      int n_stage = total < FO_STAGES ? total : FO_STAGES;
      for (int g = 0; g < n_stage; ++g) load_stage(g);
      load_w(0);
      int n_w = 1;
      bool ok = true;
      for (int g = 1; g < total; ++g) {
        // The MMAs of head g-1 are done: the W_out buffer and the stage of
        // head g-1 (= that of head g+2) are free -- after the stores of the
        // block's output staged there, if head g-1 was a block's last.
        const bool edge = g % heads == 0;
        if (!mbar_wait_bounded(m_done, (uint32_t)((g - 1) & 1), err_word,
                               VI_DEV_ERR_MMA_TIMEOUT) ||
            (edge && !store_item(g / heads - 1))) {
          ok = false;
          break;
        }
        if (edge) bulk_wait_read_le1();        // the W_out buffer's boxes have been read
        load_w(g);
        ++n_w;
        if (edge) bulk_wait_read_all();        // and the stage's
        if (g + 2 < total) {
          load_stage(g + 2);
          ++n_stage;
        }
      }
      if (ok && store_item(my_items - 1)) bulk_wait_read_all();
      // Every copy issued lands before the CTA may end (on an error path the
      // consumers may have stopped waiting for them).
      for (int s = 0; s < FO_STAGES && s < n_stage; ++s) {
        const int loads = (n_stage - s + FO_STAGES - 1) / FO_STAGES;
        mbar_wait_bounded(bars + 8 * s, (uint32_t)((loads - 1) & 1), err_word,
                          VI_DEV_ERR_TMA_TIMEOUT);
      }
      mbar_wait_bounded(w_full, (uint32_t)((n_w - 1) & 1), err_word, VI_DEV_ERR_TMA_TIMEOUT);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(128, NH);
      for (int g = 0; g < total; ++g) {
        const int s = g % FO_STAGES, h = g % heads;
        // A block's first head: the previous block's accumulator has been read.
        if ((h == 0 && g > 0 &&
             !mbar_wait_bounded(tmem_empty, (uint32_t)((g / heads - 1) & 1), err_word,
                                VI_DEV_ERR_MMA_TIMEOUT)) ||
            !mbar_wait_bounded(o_full0 + 8 * s, (uint32_t)((g / FO_STAGES) & 1), err_word,
                               VI_DEV_ERR_MMA_TIMEOUT) ||
            !mbar_wait_bounded(w_full, (uint32_t)(g & 1), err_word, VI_DEV_ERR_TMA_TIMEOUT))
          break;
        tc_fence_after();
        const uint64_t ad =
            umma_desc_kmajor_sw128(base + (uint32_t)s * Lay::STAGE + Lay::OFF_Q, 1024u);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint64_t bd = umma_desc_kmajor_sw128(sW + (uint32_t)(j * NH) * FA_ROW_BYTES, 1024u);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)   // K = 16 per MMA: 32 bytes along the swizzled rows
            umma_bf16(tmem_base + (uint32_t)(j * NH), ad + 2u * ks, bd + 2u * ks, idesc,
                      (h | ks) != 0 ? 1u : 0u);
        }
        umma_commit(m_done);                 // frees the stage and the W_out buffer
        if (h == heads - 1) umma_commit(acc_full);   // the block's accumulator is complete
      }
      // Every MMA issued is done before TMEM is released.
      umma_commit(drain);
      mbar_wait_bounded(drain, 0, err_word, VI_DEV_ERR_MMA_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ attention
    const int q = warp & 3, c = warp >> 2;   // epilogue: TMEM lane quarter, column half
    const int G = NH / 32;                   // 32-column groups of this warp (<= FO_G_MAX)
    bool ok = true;
    int g = 0;
    for (int i = 0; i < my_items && ok; ++i) {
      int p, f0;
      item_pos(i, p, f0);
      const int clip = (f0 + 16 * warp) / LQ;  // the warp's (first) clip
      for (int h = 0; h < heads; ++h, ++g) {
        const int s = g % FO_STAGES;
        const uint32_t st = base + (uint32_t)s * Lay::STAGE;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(bars + 8 * s,
                                                       (uint32_t)((g / FO_STAGES) & 1),
                                                       err_word, VI_DEV_ERR_TMA_TIMEOUT));
        if (!ok) break;
        if (clip < N)
          fa_attend_warp<H, LQ>(st + Lay::OFF_Q, st + Lay::OFF_KW, st + Lay::OFF_VW,
                            st + Lay::OFF_KG, st + Lay::OFF_VG, warp, lane, clip, N, n_pre,
                            n_post, n_global, scale_log2);
        fence_proxy_async_smem();            // O_h is visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(o_full0 + 8 * s);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(acc_full, (uint32_t)(i & 1), err_word,
                                                     VI_DEV_ERR_MMA_TIMEOUT));
      if (!ok) break;
      tc_fence_after();
      // Group by group (32 columns): TMEM -> registers (the next group's load
      // in flight meanwhile), + b_out, -> bf16 pairs, -> row 32q + lane of the
      // output boxes in the 128-byte swizzle (chunk j of row r at j ^ (r mod
      // 8)).  The producer stores the boxes.  Loops unrolled: registers
      // indexed at compile time only.
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(c * NH);
      const int row = 32 * q + lane;
      uint32_t ra[32], rb[32];
      tmem_ld32(taddr, ra);
#pragma unroll
      for (int gg = 0; gg < FO_G_MAX; ++gg) {
        if (gg >= G) break;
        uint32_t (&r)[32] = (gg & 1) ? rb : ra;
        uint32_t (&rn)[32] = (gg & 1) ? ra : rb;
        tmem_wait_ld_dep(r);
        if (gg + 1 < G) tmem_ld32(taddr + 32u * (gg + 1), rn);
        const int col = c * NH + 32 * gg;
        const uint32_t rowb = box_addr(i, col / 64) + (uint32_t)row * FA_ROW_BYTES;
        const int j0 = (col % 64) / 8;           // first 16-byte chunk of the group
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float bv[8];                           // (the same address in every lane)
          asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                       : "=f"(bv[0]), "=f"(bv[1]), "=f"(bv[2]), "=f"(bv[3])
                       : "r"(sBias + 4u * (col + 8 * e)));
          asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                       : "=f"(bv[4]), "=f"(bv[5]), "=f"(bv[6]), "=f"(bv[7])
                       : "r"(sBias + 4u * (col + 8 * e + 4)));
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int t = 8 * e + 2 * u;           // column t of the group
            w[u] = pack2_bf16(__uint_as_float(r[t]) + bv[2 * u],
                              __uint_as_float(r[t + 1]) + bv[2 * u + 1]);
          }
          sts128(rowb + ((uint32_t)((j0 + e) ^ (row & 7)) << 4), make_uint4(w[0], w[1], w[2], w[3]));
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();              // the staging is visible to the TMA stores
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(tmem_empty);             // the next block's MMAs may start
        mbar_arrive(staged);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                 CUtensorMapDataType dt);

template <int H, int LQ>
static int fo_prepare() {
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  VI_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    VI_CUDA_TRY(cudaFuncSetAttribute(dual_attn_oproj_bf16<H, LQ>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     FoLayout<H>::SMEM));
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  return VI_OK;
}

template <int H, int LQ>
static int fo_launch(const bf16* q, const bf16* k, const bf16* v, const bf16* w_out,
                     const bf16* b_out, bf16* out, int F, int N, int P, int heads, int n_pre,
                     int n_post, int n_global, cudaStream_t stream) {
  const int C = heads * 64, NH = C / 2;
  FoMaps maps;
  const uint64_t dims[3] = {(uint64_t)C, (uint64_t)F, (uint64_t)P};
  const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)F * C * 2};
  const uint32_t boxQ[3] = {64, FA_ROWS_Q, 1}, boxW[3] = {64, FaLayout<H>::ROWS_W, 1};
  const uint32_t boxY[3] = {64, FA_ROWS_Q, 1};
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = encode_tmap(&maps.q, q, 3, dims, strides, boxQ, SW, BF) &&
            encode_tmap(&maps.k, k, 3, dims, strides, boxW, SW, BF) &&
            encode_tmap(&maps.v, v, 3, dims, strides, boxW, SW, BF) &&
            encode_tmap(&maps.y, out, 3, dims, strides, boxY, SW, BF);
  {
    const uint64_t wdims[2] = {(uint64_t)C, (uint64_t)C};
    const uint64_t wstrides[1] = {(uint64_t)C * 2};
    const uint32_t wbox[2] = {64, (uint32_t)NH};
    ok = ok && encode_tmap(&maps.w, w_out, 2, wdims, wstrides, wbox, SW, BF);
  }
  if (n_global > 0) {
    const int gs = F / n_global;
    const uint64_t gdims[3] = {(uint64_t)C, (uint64_t)n_global, (uint64_t)P};
    const uint64_t gstrides[2] = {(uint64_t)gs * C * 2, (uint64_t)F * C * 2};
    const uint32_t boxG[3] = {64, FA_NG, 1};
    ok = ok && encode_tmap(&maps.kg, k, 3, gdims, gstrides, boxG, SW, BF) &&
         encode_tmap(&maps.vg, v, 3, gdims, gstrides, boxG, SW, BF);
  } else {
    maps.kg = maps.k;
    maps.vg = maps.v;
  }
  if (!ok) return VI_ERR_CUDA;
  int st = fo_prepare<H, LQ>();
  if (st != VI_OK) return st;
  const int cpb = FA_ROWS_Q / LQ;
  const int nblk = (N + cpb - 1) / cpb;
  const int64_t n_items = (int64_t)P * nblk;
  const int sms = sm_count();
  if (sms <= 0) return VI_ERR_CUDA;
  // One persistent CTA per SM (the shared memory admits no second), each
  // with at most 2^31 / heads heads of work.
  const int64_t grid = n_items < sms ? n_items : sms;
  if ((n_items + grid - 1) / grid * heads > 0x7fffffff) return VI_ERR_UNSUPPORTED;
  uint32_t tmem_cols = 64;
  while ((int)tmem_cols < C) tmem_cols <<= 1;
  const float scale_log2 = 1.4426950408889634f / 8.0f;    // log2(e) / sqrt(64)
  unsigned int* err = device_error_word();
  if (!err) return VI_ERR_CUDA;
  dual_attn_oproj_bf16<H, LQ><<<(unsigned)grid, FO_THREADS, FoLayout<H>::SMEM, stream>>>(
      maps, b_out, N, P, heads, n_pre, n_post, n_global, scale_log2, tmem_cols, err);
  VI_LAUNCHED();
  return VI_OK;
}

bool dual_attn_fast_ok(int F, int N, int d, int n_pre, int n_post, int n_global);

// The attention fast path's shapes with at most FO_C_MAX channels.
bool dual_attn_oproj_ok(int F, int N, int d, int heads, int n_pre, int n_post, int n_global) {
  return heads >= 1 && heads * 64 <= FO_C_MAX &&
         dual_attn_fast_ok(F, N, d, n_pre, n_post, n_global);
}

int dual_attn_oproj_bf16_launch(const bf16* q, const bf16* k, const bf16* v, const bf16* w_out,
                                const bf16* b_out, bf16* out, int F, int N, int P, int heads,
                                int n_pre, int n_post, int n_global, cudaStream_t stream) {
  if (F / N == 8)
    return fo_launch<FA_HALO, 8>(q, k, v, w_out, b_out, out, F, N, P, heads, n_pre, n_post,
                                 n_global, stream);
  if (F / N == 32)
    return fo_launch<FA_HALO, 32>(q, k, v, w_out, b_out, out, F, N, P, heads, n_pre, n_post,
                                  n_global, stream);
  if (n_pre <= FA_HALO && n_post <= FA_HALO)
    return fo_launch<FA_HALO, FA_L>(q, k, v, w_out, b_out, out, F, N, P, heads, n_pre, n_post,
                                    n_global, stream);
  return fo_launch<FA_HALO_MAX, FA_L>(q, k, v, w_out, b_out, out, F, N, P, heads, n_pre, n_post,
                                      n_global, stream);
}

}  // namespace vi
