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
//   persistent CTA per SM walks its items; 14 warps:
//     warps 0-7    the attention (warp w: frames 16w .. 16w+15 of the block,
//                  one clip of 16 frames, two of 8 or half of one of 32, the
//                  same per-warp code as the attention kernel), head after
//                  head and block after block;
//     warp 8       TMA producer: per head, its stage (Q, K/V window of 8 rows
//                  each side, K/V global) into a ring of 3 stages that runs on
//                  across blocks, and the columns 64h .. 64h+63 of W_out
//                  (C rows x 128 bytes) into one buffer;
//     warp 9       TMEM allocation and the MMA thread;
//     warps 10-13  the epilogue, one per TMEM lane quarter.
//   Per head, the attention warps write O_h (128 x 64 bf16) over the Q tile
//   of its stage.  That tile's 128-byte swizzle is also the K-major operand
//   layout of tcgen05.mma, so the MMA thread accumulates
//     acc += O_h W_out[:, 64h .. 64h+63]^T
//   into TMEM straight from it (128 lanes x C fp32 columns; 2 x 4 MMAs of
//   M = 128, N = C/2, K = 16 per head).  When the MMAs of head g are done,
//   its stage and the W_out buffer are free: the producer loads the W_out
//   slice of head g+1 and the stage of head g+3.
//   After a block's last head the epilogue warps read the accumulator, add
//   b_out, round to bf16 and park the packed rows in spare TMEM columns, so
//   that the accumulator goes back to the next block's MMAs at once; then
//   they store the rows through their own staging buffers with TMA (frames
//   past the end fall outside the tensor map and are dropped).
//   The attention warps never wait for the epilogue.
// The three stages, the W_out slice and the staging fill the shared memory
// with the 8-row window: contexts above 8 frames run the attention kernel
// and the output GEMM instead.
// HBM traffic per token: q, k, v read once and out written once (4 C x 2 B),
// against 6 C x 2 B for the attention plus the output GEMM.  Every block
// re-reads W_out (C x C x 2 B) from L2.
#include <atomic>

#include "dual_attn_tile.cuh"
#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

// ---- TMEM 16-column loads and stores (the epilogue's packed rows) ----------
// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane
// (taddr.lane + i), columns taddr.col .. +15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld_dep16(uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15])
      :
      : "memory");
}
// The mirror of tmem_ld16: thread i writes lane (taddr.lane + i), columns
// taddr.col .. +15.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
// Wait until this thread's TMEM stores have completed.
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

constexpr int FO_ATTN_WARPS = 8;                  // one per 16 query rows
constexpr int FO_EPI_WARPS = 4;                   // one per TMEM lane quarter
constexpr int FO_THREADS = 32 * (FO_ATTN_WARPS + 2 + FO_EPI_WARPS);   // + producer, MMA
constexpr int FO_C_MAX = 320;                     // channels (5 heads of 64)
constexpr int FO_STAGES = 3;
constexpr int FO_H = 8;                           // window rows each side (context <= 8)
constexpr uint32_t FO_EPI_BUF = 32 * 64;          // 32 frames x 32 channels of bf16

// Shared memory: 3 stages of the attention kernel's layout (without its
// barrier) | W_out slice of one head (up to FO_C_MAX rows x 128 B) | two
// output staging buffers per epilogue warp | barriers | b_out in fp32.
struct FoLayout {
  static constexpr uint32_t STAGE = FaLayout<FO_H>::STAGE;
  static constexpr uint32_t OFF_W = FO_STAGES * STAGE;
  static constexpr uint32_t OFF_EPI = OFF_W + FO_C_MAX * FA_ROW_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_EPI + FO_EPI_WARPS * 2 * FO_EPI_BUF;
  // full[3], o_full[3], w_full, m_done, acc_full, tmem_empty, drain (8 bytes
  // each), TMEM slot
  static constexpr uint32_t OFF_BIAS = OFF_BAR + 128;
  static constexpr uint32_t SMEM = OFF_BIAS + FO_C_MAX * 4 + 1024;   // + slack for alignment
  static_assert(OFF_W % 1024 == 0 && OFF_EPI % 1024 == 0,
                "the W_out slice is 128B-swizzled, the staging 64B-swizzled");
  static_assert(SMEM <= 232448, "one CTA per SM must fit");
};

struct FoMaps {
  CUtensorMap q, k, v, kg, vg;   // as in the attention kernel
  CUtensorMap w;                 // W_out [C][C]: box of 64 input channels x C/2 rows
  CUtensorMap y;                 // out [P][F][C]: box of 32 channels x 32 frames
};

// Persistent: CTA c walks the blocks (position p, 128 frames) c, c + grid,
// ... of the video (N clips of LQ = 8, 16 or 32 frames, P positions); global
// head g of the CTA is head g % heads of its block g / heads, staged in stage
// g % 3.  tmem_cols: a power of two >= 3C/2.
template <int LQ>
__global__ void __launch_bounds__(FO_THREADS, 1)
    dual_attn_oproj_bf16(const __grid_constant__ FoMaps maps, const bf16* __restrict__ b_out,
                         int N, int P, int heads, int n_pre, int n_post, int n_global,
                         float scale_log2, uint32_t tmem_cols, unsigned int* err_word) {
  using Lay = FaLayout<FO_H>;
  using FL = FoLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sW = base + FL::OFF_W, sEpi = base + FL::OFF_EPI;
  const uint32_t bars = base + FL::OFF_BAR, sBias = base + FL::OFF_BIAS;
  const uint32_t o_full0 = bars + 8 * FO_STAGES, w_full = bars + 16 * FO_STAGES;
  const uint32_t m_done = w_full + 8, acc_full = w_full + 16, tmem_empty = w_full + 24;
  const uint32_t drain = w_full + 32, tmem_slot = w_full + 40;
  const int C = heads * 64, NH = C / 2;           // NH: N of one MMA
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < FO_STAGES; ++s) {
      mbar_init(bars + 8 * s, 1);
      mbar_init(o_full0 + 8 * s, FO_ATTN_WARPS);  // one arrive per attention warp
    }
    mbar_init(w_full, 1);
    mbar_init(m_done, 1);
    mbar_init(acc_full, 1);
    mbar_init(tmem_empty, FO_EPI_WARPS);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == FO_ATTN_WARPS + 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  if ((int)threadIdx.x < C)                       // C <= FO_C_MAX <= FO_THREADS
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(sBias + 4u * threadIdx.x),
                 "f"(__bfloat162float(b_out[threadIdx.x])));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t tmem_base;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem_base) : "r"(tmem_slot));

  if (warp == FO_ATTN_WARPS) {
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
        tma_load_3d(st + Lay::OFF_KW, &maps.k, h * 64, f0 - FO_H, p, bar);
        tma_load_3d(st + Lay::OFF_VW, &maps.v, h * 64, f0 - FO_H, p, bar);
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
      int n_stage = total < FO_STAGES ? total : FO_STAGES;
      for (int g = 0; g < n_stage; ++g) load_stage(g);
      load_w(0);
      int n_w = 1;
      for (int g = 1; g < total; ++g) {
        // The MMAs of head g-1 are done: the W_out buffer and the stage of
        // head g-1 (= that of head g+2) are free.
        if (!mbar_wait_bounded(m_done, (uint32_t)((g - 1) & 1), err_word,
                               VI_DEV_ERR_MMA_TIMEOUT))
          break;
        load_w(g);
        ++n_w;
        if (g + 2 < total) {
          load_stage(g + 2);
          ++n_stage;
        }
      }
      // Every copy issued lands before the CTA may end (on an error path the
      // consumers may have stopped waiting for them).
      for (int s = 0; s < FO_STAGES && s < n_stage; ++s) {
        const int loads = (n_stage - s + FO_STAGES - 1) / FO_STAGES;
        mbar_wait_bounded(bars + 8 * s, (uint32_t)((loads - 1) & 1), err_word,
                          VI_DEV_ERR_TMA_TIMEOUT);
      }
      mbar_wait_bounded(w_full, (uint32_t)((n_w - 1) & 1), err_word, VI_DEV_ERR_TMA_TIMEOUT);
    }
  } else if (warp == FO_ATTN_WARPS + 1) {
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
  } else if (warp < FO_ATTN_WARPS) {
    // ------------------------------------------------------------ attention
    int g = 0;
    for (int i = 0; i < my_items; ++i) {
      int p, f0;
      item_pos(i, p, f0);
      const int clip = (f0 + 16 * warp) / LQ;  // the warp's (first) clip
      bool ok = true;
      for (int h = 0; h < heads; ++h, ++g) {
        const int s = g % FO_STAGES;
        const uint32_t st = base + (uint32_t)s * Lay::STAGE;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(bars + 8 * s,
                                                       (uint32_t)((g / FO_STAGES) & 1),
                                                       err_word, VI_DEV_ERR_TMA_TIMEOUT));
        if (!ok) break;
        if (clip < N)
          fa_attend_warp<FO_H, LQ>(st + Lay::OFF_Q, st + Lay::OFF_KW, st + Lay::OFF_VW,
                                   st + Lay::OFF_KG, st + Lay::OFF_VG, warp, lane, clip, N,
                                   n_pre, n_post, n_global, scale_log2);
        fence_proxy_async_smem();            // O_h is visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(o_full0 + 8 * s);
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp q (= its index mod 4, the TMEM lane quarter it may read) writes
    // frames 32q .. 32q+31 of each block, all C channels, in two phases:
    //   1. the accumulator, 32 columns at a time (the next group's load in
    //      flight during each store), + b_out, -> bf16 pairs, -> TMEM columns
    //      C .. C + C/2 - 1 (spare beside the accumulator); then the
    //      accumulator goes back to the next block's MMAs;
    //   2. the packed rows, 16 columns (32 channels) at a time, -> one of its
    //      two staging buffers (64-byte rows, chunk i of row r at
    //      i ^ ((r >> 1) & 3)), -> one TMA store (frames past the end are
    //      dropped); a buffer is written again once its previous store has
    //      read it.
    // Loops unrolled: registers indexed at compile time only.
    const int q = warp & 3;
    const uint32_t my_buf = sEpi + (uint32_t)(warp - FO_ATTN_WARPS - 2) * 2u * FO_EPI_BUF;
    const int G = C / 32;                    // 32-channel groups
    const uint32_t t_acc = tmem_base + ((uint32_t)(32 * q) << 16);
    const uint32_t t_out = t_acc + (uint32_t)C;
    int ob = 0;
    for (int i = 0; i < my_items; ++i) {
      int p, f0;
      item_pos(i, p, f0);
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(acc_full, (uint32_t)(i & 1), err_word,
                                                     VI_DEV_ERR_MMA_TIMEOUT)))
        break;
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld32(t_acc, r);
#pragma unroll
        for (int gg = 0; gg < FO_C_MAX / 32; ++gg) {
          if (gg >= G) break;
          tmem_wait_ld_dep(r);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float bv[8];                         // (the same address in every lane)
            asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                         : "=f"(bv[0]), "=f"(bv[1]), "=f"(bv[2]), "=f"(bv[3])
                         : "r"(sBias + 4u * (32 * gg + 8 * e)));
            asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                         : "=f"(bv[4]), "=f"(bv[5]), "=f"(bv[6]), "=f"(bv[7])
                         : "r"(sBias + 4u * (32 * gg + 8 * e + 4)));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int t = 8 * e + 2 * u;         // column t of the group
              pk[4 * e + u] = pack2_bf16(__uint_as_float(r[t]) + bv[2 * u],
                                         __uint_as_float(r[t + 1]) + bv[2 * u + 1]);
            }
          }
          // r is consumed: the next group's load goes in flight during the store.
          if (gg + 1 < G) tmem_ld32(t_acc + 32u * (gg + 1), r);
          tmem_st16(t_out + 16u * gg, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty);  // the next block's MMAs may start
      {
        uint32_t pa[16], pb[16];
        tmem_ld16(t_out, pa);
#pragma unroll
        for (int gg = 0; gg < FO_C_MAX / 32; ++gg) {
          if (gg >= G) break;
          uint32_t (&pc)[16] = (gg & 1) ? pb : pa;
          uint32_t (&pn)[16] = (gg & 1) ? pa : pb;
          tmem_wait_ld_dep16(pc);
          if (gg + 1 < G) tmem_ld16(t_out + 16u * (gg + 1), pn);
          const uint32_t buf = my_buf + (uint32_t)ob * FO_EPI_BUF;
          if (lane == 0) bulk_wait_read_le1();   // the store that last read this buffer is done
          __syncwarp();
          const uint32_t row = buf + (uint32_t)lane * 64u, sw = (uint32_t)((lane >> 1) & 3);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            sts128(row + (((uint32_t)e ^ sw) << 4),
                   make_uint4(pc[4 * e], pc[4 * e + 1], pc[4 * e + 2], pc[4 * e + 3]));
          fence_proxy_async_smem();              // the writes are visible to the TMA store
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&maps.y, buf, 32 * gg, f0 + 32 * q, p);
            bulk_commit();
          }
          ob ^= 1;
        }
      }
    }
    if (lane == 0) bulk_wait_read_all();       // the staging is read before the CTA ends
  }
  tc_fence_before();
  __syncthreads();
  if (warp == FO_ATTN_WARPS + 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                 CUtensorMapDataType dt);

template <int LQ>
static int fo_prepare() {
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  VI_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    VI_CUDA_TRY(cudaFuncSetAttribute(dual_attn_oproj_bf16<LQ>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     FoLayout::SMEM));
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  return VI_OK;
}

template <int LQ>
static int fo_launch(const bf16* q, const bf16* k, const bf16* v, const bf16* w_out,
                     const bf16* b_out, bf16* out, int F, int N, int P, int heads, int n_pre,
                     int n_post, int n_global, cudaStream_t stream) {
  const int C = heads * 64, NH = C / 2;
  FoMaps maps;
  const uint64_t dims[3] = {(uint64_t)C, (uint64_t)F, (uint64_t)P};
  const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)F * C * 2};
  const uint32_t boxQ[3] = {64, FA_ROWS_Q, 1}, boxW[3] = {64, FaLayout<FO_H>::ROWS_W, 1};
  const uint32_t boxY[3] = {32, 32, 1};
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = encode_tmap(&maps.q, q, 3, dims, strides, boxQ, SW, BF) &&
            encode_tmap(&maps.k, k, 3, dims, strides, boxW, SW, BF) &&
            encode_tmap(&maps.v, v, 3, dims, strides, boxW, SW, BF) &&
            encode_tmap(&maps.y, out, 3, dims, strides, boxY, CU_TENSOR_MAP_SWIZZLE_64B, BF);
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
  int st = fo_prepare<LQ>();
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
  // The accumulator (C columns) and the epilogue's packed bf16 rows (C / 2).
  uint32_t tmem_cols = 64;
  while ((int)tmem_cols < C + C / 2) tmem_cols <<= 1;
  const float scale_log2 = 1.4426950408889634f / 8.0f;    // log2(e) / sqrt(64)
  unsigned int* err = device_error_word();
  if (!err) return VI_ERR_CUDA;
  dual_attn_oproj_bf16<LQ><<<(unsigned)grid, FO_THREADS, FoLayout::SMEM, stream>>>(
      maps, b_out, N, P, heads, n_pre, n_post, n_global, scale_log2, tmem_cols, err);
  VI_LAUNCHED();
  return VI_OK;
}

bool dual_attn_fast_ok(int F, int N, int d, int n_pre, int n_post, int n_global);

// The attention fast path's shapes with at most FO_C_MAX channels and context
// of at most FO_H frames on each side (the 8-row window: three stages, the
// W_out slice and the epilogue staging fill the shared memory).
bool dual_attn_oproj_ok(int F, int N, int d, int heads, int n_pre, int n_post, int n_global) {
  return heads >= 1 && heads * 64 <= FO_C_MAX && n_pre <= FO_H && n_post <= FO_H &&
         dual_attn_fast_ok(F, N, d, n_pre, n_post, n_global);
}

int dual_attn_oproj_bf16_launch(const bf16* q, const bf16* k, const bf16* v, const bf16* w_out,
                                const bf16* b_out, bf16* out, int F, int N, int P, int heads,
                                int n_pre, int n_post, int n_global, cudaStream_t stream) {
  if (F / N == 8)
    return fo_launch<8>(q, k, v, w_out, b_out, out, F, N, P, heads, n_pre, n_post, n_global,
                        stream);
  if (F / N == 32)
    return fo_launch<32>(q, k, v, w_out, b_out, out, F, N, P, heads, n_pre, n_post, n_global,
                         stream);
  return fo_launch<FA_L>(q, k, v, w_out, b_out, out, F, N, P, heads, n_pre, n_post, n_global,
                         stream);
}

}  // namespace vi
