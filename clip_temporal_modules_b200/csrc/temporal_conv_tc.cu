// Tensor-core path of the temporal convolution (bf16 I/O, fp32 accumulation):
// tcgen05 MMAs with accumulators in tensor memory (TMEM), operands staged by
// TMA, on sm_100a.
//
// Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
// write-up), conv-module paragraph: each clip is padded with the neighbouring
// clips' boundary frames and zeros at the video ends, then convolved along
// frames with full C -> C mixing.  With the clips adjacent in HBM this is, for
// every position p, the GEMM
//   Y_p[f, co] = b[co] + sum_t sum_ci X_p[f + t - k/2, ci] W_t[co, ci]
// of M = F frames, N = C output channels and K = k * C.
//
// Tile = (position p, block of 128 frames).  Job = (tile, or a pair of tiles
// on a CTA pair, x slab of NJ output channels).  Per job the CTA runs C/64
// K-blocks; each K-block stages, with one TMA load, the x rows
// [f0 - k/2, f0 + 128 + k/2) x 64 channels ONCE (a_rows = 127 + k rows of 128
// bytes, 128-byte swizzle), so the k taps read the same shared tile through
// descriptors whose start differs by one 128-byte row per tap: the tap shift
// costs no extra load.  The frame coordinate -1 (and F) reads as zero from
// TMA's out-of-bounds fill, which is exactly the zero padding at the two ends
// of the video.  The weights are repacked once per call so that every
// (slab, K-block, tap) tile is a contiguous NJ x 64 block in the no-swizzle
// K-major layout, fetched by a 2-D TMA box of 128-byte rows.
//
// PAIR = true (built, not dispatched: see TC_USE_PAIR): a cluster of two
// CTAs on two SMs runs tcgen05.mma.cta_group::2 with M = 256: each CTA holds
// its own 128-frame tile of x and HALF of every weight tile, and its own 128
// accumulator rows in TMEM.  Per SM this halves the weight bytes streamed
// from L2 per flop, which is what limits the one-SM form.  The even CTA's
// single thread issues the MMAs; both CTAs' TMA loads complete on the even
// CTA's barriers, commits are multicast to both CTAs, and the odd CTA's
// epilogue arrives remotely on the even CTA's accumulator-empty barrier.
//
// MT = 2 (the default where it keeps the slab width): a job covers TWO tiles
// (consecutive in position-major order) on one SM, and every weight stage
// feeds both: per K-block the CTA loads two x boxes and one set of weight
// tiles and issues 2 x 4k MMAs into two accumulators.  Weight bytes per flop,
// through L2 and through shared memory, halve; shared memory (TMA writes plus
// the tensor core's operand reads) is what limits the one-tile form.
//
// TMEM holds a ring of MT + 1 (at least 2) accumulators of NJ columns: eight
// epilogue warps (TMEM -> registers, + bias, -> bf16 -> global) drain the
// oldest while the MMAs of the next tiles fill the others.  Every CTA walks
// the K-blocks of a job starting at its own offset, so the CTAs do not all
// stream the same weight tile at once.
//
// The epilogue writes y through shared memory: per 32-channel chunk of an
// accumulator the four warps write 128 rows x 64 bytes (64-byte swizzle, so
// the 16-byte writes of eight consecutive rows hit distinct banks) into one of
// two staging buffers, and one thread stores the chunk with a TMA tensor
// store, which also drops the rows past the last frame.  Full 64-byte row
// segments reach L2 in one piece (direct 16-byte stores from every row left
// partial sectors and cost a quarter of the kernel's time).
//
// Warp roles (192 threads, one CTA per SM, persistent over jobs):
//   warp 0      TMA producer (one elected thread)
//   warp 1      TMEM allocator + MMA issuer (one thread, even CTA of a pair)
//   warps 2..5  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31
//   warps 6..13 (GroupNorm fusion only) normalise the landed x tiles
#include <atomic>
#include <mutex>

#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

constexpr int TC_M = 128;        // frames per tile = TMEM lanes per CTA
constexpr int TC_KB = 64;        // input channels per K-block
constexpr int TC_SA_MAX = 6;     // A (x) stages at most
constexpr int TC_SB_MAX = 8;     // B (w) stages at most
constexpr int TC_NJ_MAX = 160;   // a B stage holds all k taps of one K-block
constexpr int TC_EPI_WARPS = 4;          // one per TMEM lane quadrant
constexpr int TC_THREADS = 64 + 32 * TC_EPI_WARPS;   // + transform threads with NORM
constexpr int TC_XF_WARPS = 8;           // NORM: warps normalising the landed x stages
constexpr int TC_OUT_CHUNK = 128 * 64;   // staged output: 128 frames x 32 channels of bf16
constexpr int TC_TMEM_COLS = 512;
constexpr int TC_SMEM_LIMIT = 232448;   // 227 KB opt-in per CTA

// Bounded wait; cluster-scope acquire when the barrier is signalled from the
// other CTA of a pair (remote arrivals, multicast commits).
template <bool PAIR>
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, unsigned int* err,
                                        unsigned int code) {
  if constexpr (PAIR) return mbar_wait_bounded_cluster(bar, parity, err, code);
  else return mbar_wait_bounded(bar, parity, err, code);
}

struct TcPlan {
  int F, P, C, k;
  int NJ;                // output channels per job (UMMA N), multiple of 32
  int H;                 // CTAs per MMA (1, or 2 for a pair); each holds NJ/H weight rows
  int MT;                // tiles per job per CTA (1, or 2 sharing every weight stage)
  int KS;                // K-blocks per pipeline stage (1, or 2 for single-tap convs)
  int n_stage;           // stages per job = ceil(n_cb / KS)
  int n_acc;             // TMEM accumulators in the ring (MT + 1, at least 2), NJ columns each
  int n_slabs;           // C / NJ
  int n_fblk;            // ceil(F / 128)
  long long n_tiles;     // P * n_fblk
  long long n_jobs;      // ceil(n_tiles / (H * MT)) * n_slabs
  int n_cb;              // C / 64
  int a_rows;            // 127 + k
  int a_tile;            // bytes of one tile's x box (a_rows x 128 B), 1024-aligned
  int a_stage;           // bytes per A stage = KS * MT * a_tile
  int b_rows;            // weight rows per CTA per tap = NJ / H
  int b_tap;             // bytes of one tap's block = b_rows * 128
  int b_kb;              // weight bytes of one K-block = k * b_tap (all taps)
  int b_stage;           // bytes per B stage = KS * b_kb
  int sa;                // A stages
  int sb;                // B stages
  int smem;              // dynamic shared memory bytes
};

struct TcArgs {
  const float* coef;     // NORM: per-channel (m_c, a_c, beta_c, 0) of the GroupNorm
  const bf16* bias;
  bf16* y;
  unsigned int* err;
  int x_off;             // row of output frame 0 in the x map (k/2 for a shard with halos)
};

// Ring depths (measured on B200 at F = 1024): with one tile per job and
// C <= 640 three x stages and two weight stages beat two and three (1.48 vs
// 1.53 ms at C = 320); at C = 1280 two x stages and as many weight stages as
// fit are best.  With the GroupNorm transform, three x stages.  Two tiles per
// job: two stages of each.  sb_pref / sa_pref / mt_pref override (0 = default).
static int g_tc_sb_pref = 0, g_tc_sa_pref = 0;
static std::atomic<int> g_tc_mt_pref{0};

static bool tc_plan(int F, int P, int C, int k, bool pair, TcPlan& pl, bool norm = false,
                    int mt = 1, int ks = 1) {
  if (k < 1 || k % 2 == 0 || 127 + k > 256 || C % TC_KB != 0) return false;
  if (mt != 1 && (mt != 2 || pair)) return false;
  if (ks != 1 && (ks != 2 || pair || norm)) return false;
  const int H = pair ? 2 : 1;
  const int n_acc = mt + 1 > 2 ? mt + 1 : 2;
  const int a_rows = 127 + k;
  const int a_tile = ((a_rows * 128 + 1023) / 1024) * 1024;
  const int a_stage = ks * mt * a_tile;
  const int fixed = 1024 /* align slack */ + 2 * TC_OUT_CHUNK /* output staging */ + 4 * C +
                    64 /* bias, padded */ + 512 /* bars */ +
                    (norm ? 16 * C : 0) /* GroupNorm coefficients */;
  // Widest slab (<= 160 output channels, a multiple of 32 dividing C) whose
  // all-tap weight stages leave room for at least two of each ring.
  for (int nj = TC_NJ_MAX; nj >= 32; nj -= 32) {
    if (C % nj != 0 || (nj / H) % 8 != 0 || n_acc * nj > TC_TMEM_COLS) continue;
    const int b_stage = ks * k * (nj / H) * 128;
    const bool few_k = C <= 640 || norm;
    int sa = g_tc_sa_pref > 0 ? g_tc_sa_pref : (mt == 2 ? 2 : few_k ? 3 : 2);
    if (sa > TC_SA_MAX) sa = TC_SA_MAX;
    int sb = g_tc_sb_pref > 0 ? g_tc_sb_pref : (mt == 2 ? 2 : few_k ? 2 : TC_SB_MAX);
    const int sb_fit = (TC_SMEM_LIMIT - fixed - sa * a_stage) / b_stage;
    if (sb > sb_fit) sb = sb_fit;
    if (sb < 2) {            // not enough room: fall back to the minimum x ring
      sa = 2;
      sb = (TC_SMEM_LIMIT - fixed - sa * a_stage) / b_stage;
      if (sb > TC_SB_MAX) sb = TC_SB_MAX;
    }
    if (sb < 2) continue;
    pl.F = F; pl.P = P; pl.C = C; pl.k = k;
    pl.NJ = nj;
    pl.H = H;
    pl.MT = mt;
    pl.KS = ks;
    pl.n_acc = n_acc;
    pl.n_slabs = C / nj;
    pl.n_fblk = (F + TC_M - 1) / TC_M;
    pl.n_tiles = (long long)P * pl.n_fblk;
    pl.n_jobs = ((pl.n_tiles + H * mt - 1) / (H * mt)) * pl.n_slabs;
    pl.n_cb = C / TC_KB;
    pl.n_stage = (pl.n_cb + ks - 1) / ks;
    pl.a_rows = a_rows;
    pl.a_tile = a_tile;
    pl.a_stage = a_stage;
    pl.b_rows = nj / H;
    pl.b_tap = pl.b_rows * 128;
    pl.b_kb = k * pl.b_tap;
    pl.b_stage = b_stage;
    pl.sa = sa;
    pl.sb = sb;
    pl.smem = fixed + sa * a_stage + sb * b_stage;
    return pl.smem <= TC_SMEM_LIMIT;
  }
  return false;
}

template <bool PAIR, bool NORM>
__global__ void __launch_bounds__(TC_THREADS + (NORM ? 32 * TC_XF_WARPS : 0), 1)
    temporal_conv_tc_kernel(const __grid_constant__ CUtensorMap tmx,
                            const __grid_constant__ CUtensorMap tmw,
                            const __grid_constant__ CUtensorMap tmy, const TcPlan pl,
                            const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sA = base;
  const uint32_t sB = sA + pl.sa * pl.a_stage;
  const uint32_t sOut = sB + pl.sb * pl.b_stage;       // 2 staging buffers, 1024-aligned
  const uint32_t sBias = sOut + 2 * TC_OUT_CHUNK;
  const uint32_t sBar = sBias + ((4 * pl.C + 63) / 64) * 64;
  // barrier block: a_full[SA] a_empty[SA] b_full[SB] b_empty[SB] acc_full[4] acc_empty[4] drain tmem_slot
  const uint32_t a_full = sBar, a_empty = a_full + 8 * TC_SA_MAX;
  const uint32_t b_full = a_empty + 8 * TC_SA_MAX, b_empty = b_full + 8 * TC_SB_MAX;
  const uint32_t acc_full = b_empty + 8 * TC_SB_MAX, acc_empty = acc_full + 32;
  const uint32_t drain = acc_empty + 32, tmem_slot = drain + 8;
  const uint32_t a_ready = tmem_slot + 8;      // NORM: x stage normalised [SA]
  const uint32_t sCoef = sBar + 512;           // NORM: float4 per channel
  float* bias_s = reinterpret_cast<float*>(smem_raw + (sBias - smem_u32(smem_raw)));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const long long cluster_id = PAIR ? blockIdx.x / 2 : blockIdx.x;
  const long long n_clusters = PAIR ? gridDim.x / 2 : gridDim.x;
  // In a pair, the full barriers and the accumulator-empty barrier that count
  // both CTAs live in the even CTA; these are their cluster addresses.
  const uint32_t lead_a_full = PAIR ? mapa_shared(a_full, 0) : a_full;
  const uint32_t lead_b_full = PAIR ? mapa_shared(b_full, 0) : b_full;
  const uint32_t lead_acc_empty = PAIR ? mapa_shared(acc_empty, 0) : acc_empty;

  if (threadIdx.x == 0) {
    for (int i = 0; i < pl.sa; ++i) { mbar_init(a_full + 8 * i, PAIR ? 2 : 1); mbar_init(a_empty + 8 * i, 1); }
    for (int i = 0; i < pl.sb; ++i) { mbar_init(b_full + 8 * i, PAIR ? 2 : 1); mbar_init(b_empty + 8 * i, 1); }
    for (int i = 0; i < pl.n_acc; ++i) {
      mbar_init(acc_full + 8 * i, 1);
      mbar_init(acc_empty + 8 * i, PAIR ? 2 * TC_EPI_WARPS : TC_EPI_WARPS);
    }
    mbar_init(drain, 1);
    if (NORM)
      for (int i = 0; i < pl.sa; ++i) mbar_init(a_ready + 8 * i, TC_XF_WARPS);
    fence_barrier_init();
  }
  for (int c = threadIdx.x; c < pl.C; c += blockDim.x) bias_s[c] = to_f32(args.bias[c]);
  if constexpr (NORM) {
    float4* coef_s = reinterpret_cast<float4*>(smem_raw + (sCoef - smem_u32(smem_raw)));
    // Channel cb*64 + 8c + e sits at slot cb*64 + 8e + c: the transform threads
    // of one quarter-warp, which hold the 8 different c of a K-block, then
    // read 8 consecutive slots (no bank conflict).
    for (int ch = threadIdx.x; ch < pl.C; ch += blockDim.x)
      coef_s[(ch & ~63) + (ch & 7) * 8 + ((ch >> 3) & 7)] =
          reinterpret_cast<const float4*>(args.coef)[ch];
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, TC_TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TC_TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();      // barriers of both CTAs initialised
  tc_fence_after();
  uint32_t tmem_base;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem_base) : "r"(tmem_slot));

  const int halo = pl.k / 2;
  const int cb_rot = (int)(cluster_id % pl.n_cb);
  // Equal x and w rings (the two-tile form): one barrier pair per stage covers
  // both, so a K-block costs one wait and one commit.
  const bool uni = !PAIR && pl.sa == pl.sb;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Ring positions as (stage, phase) counters: no division in the loop.
      int sa = 0, pa = 0, sbi = 0, pb = 0;
      bool a_used = false, b_used = false;         // first pass over a ring needs no wait
      bool ok = true;
      for (long long job = cluster_id; job < pl.n_jobs && ok; job += n_clusters) {
        const int slab = (int)(job % pl.n_slabs);
        const long long tile0 = (job / pl.n_slabs) * (pl.H * pl.MT) + rank;
        // Frame row and position of each tile of the job; p == P past the
        // last tile, which reads as zeros.
        int frow[2], pos[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const long long tile = tile0 + m;
          frow[m] = (int)(tile % pl.n_fblk) * TC_M - halo + args.x_off;
          pos[m] = (int)(tile / pl.n_fblk);
        }
        int wrow = (slab * pl.n_cb * pl.k * pl.H + (int)rank) * pl.b_rows;   // row of (slab, cb 0, t 0)
        const int wrow_cb = pl.k * pl.H * pl.b_rows, wrow_t = pl.H * pl.b_rows;
        for (int is = 0; is < pl.n_stage && ok; ++is) {
          // Stage `is` holds K-blocks kb0 .. kb0 + nkb - 1 of the job (in the
          // CTA's rotated order); only a job's last stage can hold fewer than KS.
          const int kb0 = is * pl.KS;
          const int nkb = min(pl.KS, pl.n_cb - kb0);
          if (a_used && !tc_wait<PAIR>(a_empty + 8 * sa, (uint32_t)(pa ^ 1), args.err,
                                       VI_DEV_ERR_TMA_TIMEOUT)) { ok = false; break; }
          const uint32_t dst = sA + sa * pl.a_stage;
          const uint32_t a_bar = a_full + 8 * sa;
          if constexpr (PAIR) {
            const int cb = (kb0 + cb_rot) % pl.n_cb;
            mbar_arrive_expect_tx_cluster(lead_a_full + 8 * sa, (uint32_t)pl.a_rows * 128u);
            tma_load_3d_pair(dst, &tmx, cb * TC_KB, frow[0], pos[0], lead_a_full + 8 * sa);
          } else {
            mbar_arrive_expect_tx(a_bar, (uint32_t)nkb * ((uint32_t)(pl.MT * pl.a_rows) * 128u +
                                                          (uni ? (uint32_t)pl.b_kb : 0u)));
            for (int kb = 0; kb < nkb; ++kb) {
              const int cb = (kb0 + kb + cb_rot) % pl.n_cb;
              const uint32_t d = dst + (uint32_t)(kb * pl.MT) * pl.a_tile;
              tma_load_3d(d, &tmx, cb * TC_KB, frow[0], pos[0], a_bar);
              if (pl.MT == 2) tma_load_3d(d + pl.a_tile, &tmx, cb * TC_KB, frow[1], pos[1], a_bar);
            }
          }
          if (++sa == pl.sa) { sa = 0; pa ^= 1; a_used = true; }
          // One B stage = this CTA's weight blocks of every tap of the stage's K-blocks.
          uint32_t b_bar = a_bar;                  // shared stage: same barrier as x
          if (!uni) {
            if (b_used && !tc_wait<PAIR>(b_empty + 8 * sbi, (uint32_t)(pb ^ 1), args.err,
                                         VI_DEV_ERR_TMA_TIMEOUT)) { ok = false; break; }
            b_bar = PAIR ? lead_b_full + 8 * sbi : b_full + 8 * sbi;
            if constexpr (PAIR) mbar_arrive_expect_tx_cluster(b_bar, (uint32_t)pl.b_stage);
            else mbar_arrive_expect_tx(b_bar, (uint32_t)(nkb * pl.b_kb));
          }
          for (int kb = 0; kb < nkb; ++kb) {
            const int cb = (kb0 + kb + cb_rot) % pl.n_cb;
            for (int t = 0; t < pl.k; ++t) {
              // Row of this CTA's weight block in the packed [..][128 B] view.
              const int row = wrow + cb * wrow_cb + t * wrow_t;
              const uint32_t dstb = sB + sbi * pl.b_stage + (uint32_t)(kb * pl.k + t) * pl.b_tap;
              if constexpr (PAIR) tma_load_2d_pair(dstb, &tmw, 0, row, b_bar);
              else tma_load_2d(dstb, &tmw, 0, row, b_bar);
            }
          }
          if (++sbi == pl.sb) { sbi = 0; pb ^= 1; b_used = true; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(TC_M * pl.H, pl.NJ);
      const uint32_t lbo_b = (uint32_t)pl.b_rows * 16u;
      // Descriptors of stage 0; stage s adds s * stage_bytes / 16 to the start field.
      const uint64_t ad_base = umma_desc_kmajor_sw128(sA, 1024u);
      const uint64_t bd_base = umma_desc_kmajor_noswizzle(sB, lbo_b, 128u);
      const uint32_t a_st16 = (uint32_t)pl.a_stage >> 4, b_st16 = (uint32_t)pl.b_stage >> 4;
      const uint32_t bt16 = (uint32_t)pl.b_tap >> 4;  // one tap's block in w
      const uint32_t bk16 = (2u * lbo_b) >> 4;     // one K step of 16 in w
      const uint32_t at16 = (uint32_t)pl.a_tile >> 4;  // second tile of an x stage
      int sa = 0, pa = 0, sbi = 0, pb = 0;
      // Accumulator ring: n_acc slots of NJ columns, one per tile, in order.
      int slot = 0, pslot = 0;
      bool slot_used = false;
      bool ok = true;
      for (long long job = cluster_id; job < pl.n_jobs && ok; job += n_clusters) {
        // This job's accumulator slots and the parity of their last release.
        int js[2], jp[2];
        bool ju[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          js[m] = slot; jp[m] = pslot; ju[m] = slot_used;
          if (m < pl.MT && ++slot == pl.n_acc) { slot = 0; pslot ^= 1; slot_used = true; }
        }
        for (int is = 0; is < pl.n_stage && ok; ++is) {
          const int nkb = min(pl.KS, pl.n_cb - is * pl.KS);
          const bool last_stage = is == pl.n_stage - 1;
          if (!tc_wait<PAIR>((NORM ? a_ready : a_full) + 8 * sa, (uint32_t)pa, args.err,
                             VI_DEV_ERR_TMA_TIMEOUT) ||
              (!uni &&
               !tc_wait<PAIR>(b_full + 8 * sbi, (uint32_t)pb, args.err, VI_DEV_ERR_TMA_TIMEOUT))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bd_stage = bd_base + (uint64_t)(sbi * b_st16);
          const uint64_t ad_stage = ad_base + (uint64_t)(sa * a_st16);
          for (int kb = 0; kb < nkb && ok; ++kb) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              if (m >= pl.MT) break;
              if (is == 0 && kb == 0) {
                // The slot must have been drained by the epilogue of its last job.
                if (ju[m] && !tc_wait<PAIR>(acc_empty + 8 * js[m], (uint32_t)(jp[m] ^ 1),
                                            args.err, VI_DEV_ERR_MMA_TIMEOUT)) { ok = false; break; }
                tc_fence_after();
              }
              const uint32_t d_tmem = tmem_base + (uint32_t)(js[m] * pl.NJ);
              // k taps x 4 K steps = 4k MMAs back to back per tile and K-block;
              // a stage queues KS x MT x 4k of them (24 for k = 3 with two
              // tiles, 16 for k = 1 with two tiles and two K-blocks): enough
              // tensor work to hide the stage's wait/commit.
              const uint64_t ad_tile = ad_stage + (uint64_t)((kb * pl.MT + m) * at16);
              const uint64_t bd_kb = bd_stage + (uint64_t)(kb * pl.k * bt16);
              uint32_t acc = (is > 0 || kb > 0) ? 1u : 0u;
              for (int t = 0; t < pl.k; ++t) {
                // Tap t: the x tile shifted down by t rows of 128 B (8 units of 16 B).
                const uint64_t ad = ad_tile + (uint64_t)(8u * t);
                const uint64_t bd = bd_kb + (uint64_t)(t * bt16);
                // K steps of 16: +32 B inside the swizzled x rows, +2 columns of 8 in w.
                if constexpr (PAIR) {
                  umma_bf16_pair(d_tmem, ad, bd, idesc, acc);
                  umma_bf16_pair(d_tmem, ad + 2u, bd + bk16, idesc, 1u);
                  umma_bf16_pair(d_tmem, ad + 4u, bd + 2u * bk16, idesc, 1u);
                  umma_bf16_pair(d_tmem, ad + 6u, bd + 3u * bk16, idesc, 1u);
                } else {
                  umma_bf16(d_tmem, ad, bd, idesc, acc);
                  umma_bf16(d_tmem, ad + 2u, bd + bk16, idesc, 1u);
                  umma_bf16(d_tmem, ad + 4u, bd + 2u * bk16, idesc, 1u);
                  umma_bf16(d_tmem, ad + 6u, bd + 3u * bk16, idesc, 1u);
                }
                acc = 1u;
              }
              if (last_stage && kb == nkb - 1) {      // accumulator ready for the epilogue
                if constexpr (PAIR) umma_commit_pair_mc(acc_full + 8 * js[m], 0x3);
                else umma_commit(acc_full + 8 * js[m]);
              }
            }
          }
          if (!ok) break;
          if constexpr (PAIR) {
            umma_commit_pair_mc(b_empty + 8 * sbi, 0x3);
            umma_commit_pair_mc(a_empty + 8 * sa, 0x3);
          } else {
            if (!uni) umma_commit(b_empty + 8 * sbi);   // frees the w stage when these MMAs finish
            umma_commit(a_empty + 8 * sa);        // frees the x stage (and the w stage if shared)
          }
          if (++sbi == pl.sb) { sbi = 0; pb ^= 1; }
          if (++sa == pl.sa) { sa = 0; pa ^= 1; }
        }
      }
      // Every MMA this thread issued must finish before TMEM is released.
      if constexpr (PAIR) umma_commit_pair_mc(drain, 0x3);
      else umma_commit(drain);
      tc_wait<PAIR>(drain, 0, args.err, VI_DEV_ERR_MMA_TIMEOUT);
    }
  } else if (warp >= 2 + TC_EPI_WARPS) {
    // ------------------------------------------------------------ transform (NORM)
    // Normalise each landed x stage in place, x -> (x - m_c) a_c + beta_c,
    // then hand it to the MMA.  Rows outside [0, F) stay zero: the conv pads
    // the normalised sequence with zeros.  128B swizzle: the 16-byte chunk of
    // channels [8c, 8c+8) of row r sits at chunk c ^ (r mod 8).
    if constexpr (NORM) {
      const float4* coef_s = reinterpret_cast<const float4*>(smem_raw + (sCoef - smem_u32(smem_raw)));
      uint4* stage0 = reinterpret_cast<uint4*>(smem_raw + (sA - smem_u32(smem_raw)));
      // Thread tt always handles physical chunk pc of rows r0, r0 + 4 TC_XF_WARPS,
      // ...; all those rows share r mod 8, so the logical chunk (its 8
      // channels) is fixed.
      const int tt = threadIdx.x - TC_THREADS;
      const int pc = tt & 7, r0 = tt >> 3;
      const int c = pc ^ (r0 & 7);
      int sa = 0, pa = 0;
      bool ok = true;
      for (long long job = cluster_id; job < pl.n_jobs && ok; job += n_clusters) {
        const long long tile0 = (job / pl.n_slabs) * (pl.H * pl.MT) + rank;
        int f_first[2];                            // frame of row 0 of each tile's x box
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) f_first[mt] = (int)((tile0 + mt) % pl.n_fblk) * TC_M - halo;
        for (int ib = 0; ib < pl.n_cb && ok; ++ib) {
          const int cb = (ib + cb_rot) % pl.n_cb;
          float m[8], a[8], bt[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 k4 = coef_s[cb * TC_KB + e * 8 + c];
            m[e] = k4.x; a[e] = k4.y; bt[e] = k4.z;
          }
          if (!mbar_wait_bounded(a_full + 8 * sa, (uint32_t)pa, args.err, VI_DEV_ERR_TMA_TIMEOUT)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            if (mt >= pl.MT) break;
            uint4* st = stage0 + (size_t)sa * (pl.a_stage / 16) + (size_t)mt * (pl.a_tile / 16);
            for (int r = r0; r < pl.a_rows; r += 4 * TC_XF_WARPS) {
              const int f = f_first[mt] + r;
              if (f < 0 || f >= pl.F) continue;
              float v[8];
              unpack(st[r * 8 + pc], v);
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = fmaf(v[e] - m[e], a[e], bt[e]);
              st[r * 8 + pc] = pack(v);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(a_ready + 8 * sa);
          if (++sa == pl.sa) { sa = 0; pa ^= 1; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                      // TMEM lane quadrant of this warp
    const int m = 32 * q + lane;                 // frame within the tile
    const bool leader = warp == 2 && lane == 0;  // issues the TMA stores
    // Row m of a staging buffer: 64 bytes; its 16-byte chunk i sits at
    // i ^ ((m >> 1) & 3) (64-byte swizzle, buffers 1024-aligned).
    const uint32_t row_off = (uint32_t)m * 64u;
    const uint32_t swz = (uint32_t)((m >> 1) & 3);
    int ob = 0;                                  // staging buffer of the next chunk
    int buf = 0, pacc = 0;                       // accumulator ring, as the MMA issuer walks it
    bool ok = true;
    for (long long job = cluster_id; job < pl.n_jobs && ok; job += n_clusters) {
      const int slab = (int)(job % pl.n_slabs);
      const float* bs = bias_s + slab * pl.NJ;
      for (int mt = 0; mt < pl.MT; ++mt) {
        // The four warps take the (bounded) wait's outcome together, so that
        // none of them is left at the staging barriers below.
        bool got = tc_wait<PAIR>(acc_full + 8 * buf, (uint32_t)pacc, args.err,
                                 VI_DEV_ERR_MMA_TIMEOUT);
        got = named_bar_and(1, 32 * TC_EPI_WARPS, got);
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        const long long tile = (job / pl.n_slabs) * (pl.H * pl.MT) + rank + mt;
        const int fb = (int)(tile % pl.n_fblk);
        const int p = (int)(tile / pl.n_fblk);
        const bool tile_ok = tile < pl.n_tiles;
        for (int c0 = 0; c0 < pl.NJ; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * pl.NJ + c0), r);
          tmem_wait_ld_dep(r);
          const uint32_t stage = sOut + (uint32_t)ob * TC_OUT_CHUNK;
          if (leader) bulk_wait_read_le1();   // the store that last read this buffer is done
          named_bar_sync(1, 32 * TC_EPI_WARPS);
          if (tile_ok) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack2_bf16(__uint_as_float(r[2 * i]) + bs[c0 + 2 * i],
                                 __uint_as_float(r[2 * i + 1]) + bs[c0 + 2 * i + 1]);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              sts128(stage + row_off + (((uint32_t)i ^ swz) << 4),
                     make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]));
          }
          fence_proxy_async_smem();           // the writes are visible to the TMA store
          named_bar_sync(1, 32 * TC_EPI_WARPS);
          if (leader && tile_ok) {
            // Rows past the last frame fall outside the tensor map and are dropped.
            tma_store_3d(&tmy, stage, slab * pl.NJ + c0, fb * TC_M, p);
            bulk_commit();
          }
          ob ^= 1;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(lead_acc_empty + 8 * buf);
          else mbar_arrive(acc_empty + 8 * buf);
        }
        if (++buf == pl.n_acc) { buf = 0; pacc ^= 1; }
      }
    }
    if (leader) bulk_wait_all();                 // every output chunk has reached global memory
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();        // the pair is done with each other's memory
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, TC_TMEM_COLS);
    else tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

// w [C_out][C_in][k] -> [slab][cb][t][h][8 columns][NJ/H][8]: for each (slab,
// K-block, tap, CTA of the pair) an NJ/H x 64 K-major block in the no-swizzle
// layout, contiguous.
__global__ void temporal_conv_pack_w(const bf16* __restrict__ w, bf16* __restrict__ wpk, int C,
                                     int k, int NJ, int H) {
  const long long total = (long long)C * C * k;
  const int n_cb = C / TC_KB, R = NJ / H;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int e = (int)(i & 7);
    long long r = i >> 3;
    const int n = (int)(r % R); r /= R;
    const int col = (int)(r % 8); r /= 8;
    const int h = (int)(r % H); r /= H;
    const int t = (int)(r % k); r /= k;
    const int cb = (int)(r % n_cb);
    const int slab = (int)(r / n_cb);
    const int co = slab * NJ + h * R + n, ci = cb * TC_KB + col * 8 + e;
    wpk[i] = w[((size_t)co * C + ci) * k + t];
  }
}

bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                 CUtensorMapDataType dt);

// The CTA-pair form is correct but, measured on B200, slower than the
// one-SM form at every workload here, so the dispatcher takes the one-SM form.
constexpr bool TC_USE_PAIR = false;
// Tiles per job of the one-SM form when the plan fits (2: every weight stage
// feeds two 128-frame tiles).
constexpr int TC_MT_DEFAULT = 2;

// Tiles per job of the one-SM form: 0 = automatic, 1 or 2 = that form where
// its plan fits.  Returns the previous setting.
int conv_set_tiles_per_job(int mt) { return g_tc_mt_pref.exchange(mt); }

bool temporal_conv_tc_ok(int F, int P, int C, int k) {
  TcPlan pl;
  return F > 0 && P > 0 && tc_plan(F, P, C, k, TC_USE_PAIR, pl);
}

bool temporal_conv_tc_norm_ok(int F, int P, int C, int k) {
  TcPlan pl;
  return F > 0 && P > 0 && tc_plan(F, P, C, k, false, pl, true);
}

template <bool PAIR, bool NORM>
static int tc_launch(const CUtensorMap& tmx, const CUtensorMap& tmw, const CUtensorMap& tmy,
                     const TcPlan& pl, const TcArgs& a, cudaStream_t stream) {
  static std::mutex mu;
  static bool attr_done[64] = {false};
  int dev = 0;
  VI_CUDA_TRY(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && !attr_done[dev]) {
      VI_CUDA_TRY(cudaFuncSetAttribute(temporal_conv_tc_kernel<PAIR, NORM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TC_SMEM_LIMIT));
      attr_done[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(TC_THREADS + (NORM ? 32 * TC_XF_WARPS : 0));
  cfg.dynamicSmemBytes = (size_t)pl.smem;
  cfg.stream = stream;
  long long grid;
  if constexpr (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2 * sm_count());
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, temporal_conv_tc_kernel<PAIR, NORM>, &cfg) !=
            cudaSuccess ||
        clusters < 1)
      clusters = sm_count() / 2;
    grid = clusters;
    if (grid > pl.n_jobs) grid = pl.n_jobs;
    grid *= 2;
  } else {
    grid = sm_count();
    if (grid > pl.n_jobs) grid = pl.n_jobs;
  }
  cfg.gridDim = dim3((unsigned)grid);
  VI_CUDA_TRY(cudaLaunchKernelEx(&cfg, temporal_conv_tc_kernel<PAIR, NORM>, tmx, tmw, tmy, pl, a));
  note_launch();
  return VI_OK;
}

// coef != nullptr: normalise x on the fly with the GroupNorm coefficients
// (m_c, a_c, beta_c) before the contraction (fused GroupNorm -> conv).
static int tc_run(const bf16* x, int x_rows, int x_off, const bf16* w, const bf16* b, bf16* y,
                  int F, int P, int C, int k, cudaStream_t stream, const float* coef) {
  TcPlan pl;
  const bool norm = coef != nullptr;
  const bool pair = !norm && TC_USE_PAIR && tc_plan(F, P, C, k, true, pl);
  if (!pair) {
    if (!tc_plan(F, P, C, k, false, pl, norm)) return VI_ERR_UNSUPPORTED;
    // Two tiles per job when that plan keeps the slab width (a narrower MMA
    // N costs more than the weight traffic it saves).
    const int pref = g_tc_mt_pref.load(std::memory_order_relaxed);
    const int mt = pref > 0 ? pref : TC_MT_DEFAULT;
    TcPlan pl2;
    if (mt == 2 && tc_plan(F, P, C, k, false, pl2, norm, 2) && pl2.NJ >= pl.NJ) pl = pl2;
    // Single tap: two K-blocks per stage where they fit at the same width, so
    // a stage still queues 16 MMAs per wait/commit.
    if (k == 1 && pl.MT == 2 && !norm && tc_plan(F, P, C, k, false, pl2, false, 2, 2) &&
        pl2.NJ >= pl.NJ)
      pl = pl2;
  }
  unsigned int* err = device_error_word();
  if (!err) return VI_ERR_CUDA;
  // x as [P][x_rows][C]: box of 64 channels x a_rows frames x 1 position, 128B swizzle.
  CUtensorMap tmx, tmw, tmy;
  {
    // y as [P][F][C]: box of 32 channels x 128 frames x 1 position, 64B swizzle.
    const uint64_t dims[3] = {(uint64_t)C, (uint64_t)F, (uint64_t)P};
    const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)F * C * 2};
    const uint32_t box[3] = {32, (uint32_t)TC_M, 1};
    if (!encode_tmap(&tmy, y, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      return VI_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)C, (uint64_t)x_rows, (uint64_t)P};
    const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)x_rows * C * 2};
    const uint32_t box[3] = {(uint32_t)TC_KB, (uint32_t)pl.a_rows, 1};
    if (!encode_tmap(&tmx, x, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      return VI_ERR_CUDA;
  }
  const size_t wbytes = (size_t)C * C * k * sizeof(bf16);
  void* wpk = nullptr;
  VI_CUDA_TRY(scratch_alloc(&wpk, wbytes, stream));
  int st = VI_OK;
  {
    // Packed weights viewed as rows of 128 bytes; one box = one CTA's block.
    const uint64_t dims[2] = {64, (uint64_t)C * C * k / 64};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, (uint32_t)pl.b_rows};
    if (!encode_tmap(&tmw, wpk, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      st = VI_ERR_CUDA;
  }
  if (st == VI_OK) {
    const long long total = (long long)C * C * k;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
    temporal_conv_pack_w<<<blocks, 256, 0, stream>>>(w, static_cast<bf16*>(wpk), C, k, pl.NJ,
                                                     pl.H);
    if (cudaGetLastError() != cudaSuccess) st = VI_ERR_CUDA; else note_launch();
  }
  if (st == VI_OK) {
    TcArgs a{coef, b, y, err, x_off};
    st = norm ? tc_launch<false, true>(tmx, tmw, tmy, pl, a, stream)
              : pair ? tc_launch<true, false>(tmx, tmw, tmy, pl, a, stream)
                     : tc_launch<false, false>(tmx, tmw, tmy, pl, a, stream);
  }
  if (scratch_free(wpk, stream) != cudaSuccess && st == VI_OK) st = VI_ERR_CUDA;
  return st;
}

int temporal_conv_bf16_tc(const bf16* x, const bf16* w, const bf16* b, bf16* y, int F, int P,
                          int C, int k, cudaStream_t stream, const float* coef) {
  return tc_run(x, F, 0, w, b, y, F, P, C, k, stream, coef);
}

// One shard of a video cut along frames: x_ext [P][F_loc + 2(k/2)][C] holds
// the k/2 frames before the shard (zeros at the start of the video), the
// shard's frames and the k/2 frames after it (zeros at the end); y is
// [P][F_loc][C].
int temporal_conv_bf16_tc_shard(const bf16* x_ext, const bf16* w, const bf16* b, bf16* y,
                                int F_loc, int P, int C, int k, cudaStream_t stream) {
  return tc_run(x_ext, F_loc + 2 * (k / 2), k / 2, w, b, y, F_loc, P, C, k, stream, nullptr);
}

}  // namespace vi
