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
// of M = F frames, N = C_out output channels and K = k * C_in.  With k = 1 the
// same kernel is a per-frame linear layer (the projections of the attention
// module), and it may then write its output channels to up to three tensors
// (q, k and v of one fused projection).
//
// Tile = (position p, block of 128 frames).  Job = (MT tiles consecutive in
// position-major order, x slab of NJ output channels).  Per job the CTA runs
// C_in/64 K-blocks; each K-block stages, with one TMA load per tile, the x
// rows [f0 - k/2, f0 + 128 + k/2) x 64 channels ONCE (a_rows = 127 + k rows of
// 128 bytes, 128-byte swizzle), so the k taps read the same shared tile
// through descriptors whose start differs by one 128-byte row per tap: the
// tap shift costs no extra load.  The frame coordinate -1 (and F) reads as
// zero from TMA's out-of-bounds fill, which is exactly the zero padding at the
// two ends of the video.  The weights are repacked once per call so that the
// k tap blocks of every (slab, K-block) are one contiguous run of k NJ x 64
// blocks in the no-swizzle K-major layout, fetched by one bulk copy.
//
// MT = 2 (the default where it keeps the slab width): every weight stage feeds
// two tiles, so the weight bytes per flop through L2 and shared memory halve.
//
// The MMA issue loop is unrolled at compile time over the taps (k = 1 and 3),
// the tiles of a job and the four K steps of a K-block, with every descriptor
// offset an immediate, and the ring layout (one shared x/w ring for two tiles
// per job) is known at compile time: the tensor pipe queues only about three
// MMAs ahead of the issuing thread, so run-time tests and address arithmetic
// between MMAs show up directly as idle pipe cycles.
//
// TMEM holds a ring of MT + 1 (at least 2) accumulators of NJ columns: the
// epilogue warps drain the oldest while the MMAs of the next tiles fill the
// others.  Every CTA walks the K-blocks of a job starting at its own offset,
// so the CTAs do not all stream the same weight block at once.
//
// Epilogue: each warp owns a TMEM lane quadrant (32 frames of the tile),
// brings its row of the accumulator into registers 32 columns at a time,
// adds the bias and packs each group to bf16 pairs (the whole row then takes
// 80 registers), releases the accumulator, and writes 64-channel chunks (32
// where the plan is narrow) into its own two 128-byte-swizzled staging
// buffers; its lane 0 stores each chunk with a TMA tensor store, which also
// drops the rows past the last frame.
//
// Warp roles (192 threads, one CTA per SM, persistent over jobs):
//   warp 0      TMA producer: lane 0 takes the ring waits, lane m loads tile
//               m's x box and lane MT the stage's weights
//   warp 1      TMEM allocator + MMA issuer (one thread)
//   warps 2..5  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31
#include <mutex>

#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

constexpr int TC_M = 128;        // frames per tile = TMEM lanes
constexpr int TC_KB = 64;        // input channels per K-block
constexpr int TC_SA_MAX = 6;     // A (x) stages at most
constexpr int TC_SB_MAX = 8;     // B (w) stages at most
constexpr int TC_NJ_MAX = 160;   // a B stage holds all k taps of one K-block
constexpr int TC_EPI_WARPS = 4;          // one per TMEM lane quadrant
constexpr int TC_THREADS = 64 + 32 * TC_EPI_WARPS;
constexpr int TC_OUT_BUF = 32 * 128;     // one staging buffer: 32 frames x 64 channels of bf16
constexpr int TC_TMEM_COLS = 512;
constexpr int TC_SMEM_LIMIT = 232448;    // 227 KB opt-in per CTA
constexpr int TC_MAX_OUT = 3;            // output tensors of one call

struct TcPlan {
  int F, P, C, k;
  int Cout;              // output channels (all output tensors together)
  int NJ;                // output channels per job (UMMA N), multiple of 32
  int MT;                // tiles per job per CTA (1, or 2 sharing every weight stage)
  int H;                 // CTAs per MMA: 1, or 2 for a CTA pair (M = 256, each holding NJ/2 weight rows)
  int b_rows;            // weight rows per CTA = NJ / H
  int n_stage;           // stages per job = n_cb (a stage is one K-block)
  int n_acc;             // TMEM accumulators in the ring (MT + 1, at least 2), NJ columns each
  int n_slabs;           // Cout / NJ
  int slabs_per_out;     // slabs of one output tensor
  int n_fblk;            // ceil(F / 128)
  int sel_lo, sel_hi0, n_sel;   // frame blocks computed per position: [0, sel_lo) and
                                // [sel_hi0, sel_hi0 + n_sel - sel_lo) (all of them by default)
  long long n_tiles;     // P * n_sel
  long long n_jobs;      // ceil(n_tiles / (H MT)) * n_slabs
  int n_cb;              // C / 64
  int a_rows;            // 127 + k
  int a_tile;            // bytes of one tile's x box (a_rows x 128 B), 1024-aligned
  int a_stage;           // bytes per A stage = MT * a_tile
  int b_tap;             // bytes of one tap's block = b_rows * 128
  int b_kb;              // weight bytes of one K-block = k * b_tap (all taps)
  int b_stage;           // bytes per B stage = b_kb
  int sa;                // A stages
  int sb;                // B stages
  int hT;                // bias tables by distance to the video ends, up to hT frames:
  int n_tab;             // (hT + 1)^2 tables of Cout floats (1 table when hT == 0)
  int wide;              // 1: the epilogue stores 64-channel chunks (else 32)
  int smem;              // dynamic shared memory bytes
};

struct TcArgs {
  const float* btab;     // fp32 bias tables [n_tab][Cout] in global memory (one table,
                         // the conv's bias, unless the GroupNorm is folded in)
  const bf16* wpk;       // packed weights
  unsigned int* err;
  int x_off;             // row of output frame 0 in the x map (k/2 for a shard with halos)
};

// Tensor maps of one launch: x as [P][x_rows][C], each output as
// [P][F][Cout/n_out] with 64-channel boxes (y) and 32-channel boxes (y32),
// and (CTA pair) the packed weights as blocks of b_rows x 128 bytes.
struct TcMaps {
  CUtensorMap x;
  CUtensorMap w;
  CUtensorMap y[TC_MAX_OUT];
  CUtensorMap y32[TC_MAX_OUT];
};

// Ring depths.  Two tiles per job: equal x and w rings (one barrier pair per
// stage), as deep as fit, at most 4.  One tile per job (measured on B200 at
// F = 1024): with C <= 640 three x stages and two weight stages beat two and
// three; at C = 1280 two x stages and as many weight stages as fit.  The
// epilogue stages 64-channel
// chunks (two 4 KB buffers per warp) where that still leaves the widest slab
// room, else 32-channel chunks (two 2 KB buffers per warp).
static bool tc_plan(int F, int P, int C, int Cout, int n_out, int k, TcPlan& pl, int hT,
                    int mt, bool pair = false) {
  if (k < 1 || k % 2 == 0 || 127 + k > 256 || C % TC_KB != 0) return false;
  if (n_out < 1 || n_out > TC_MAX_OUT || Cout <= 0 || Cout % n_out != 0) return false;
  if (mt != 1 && mt != 2) return false;
  if (pair && mt != 2) return false;
  const int H = pair ? 2 : 1;
  if (hT < 0 || hT > k / 2) return false;
  const int n_tab = (hT + 1) * (hT + 1);
  const int cpo = Cout / n_out;
  const int n_acc = mt + 1 > 2 ? mt + 1 : 2;
  const int a_rows = 127 + k;
  const int a_tile = ((a_rows * 128 + 1023) / 1024) * 1024;
  const int a_stage = mt * a_tile;
  const int base = 1024 /* align slack */ + 512 /* bars */;
  // Widest slab (<= 160 output channels, a multiple of 32 dividing each
  // output tensor's channels) whose all-tap weight stages leave room for at
  // least two of each ring.
  for (int nj = TC_NJ_MAX; nj >= 32; nj -= 32) {
    if (cpo % nj != 0 || n_acc * nj > TC_TMEM_COLS || (nj / H) % 8 != 0) continue;
    const int b_stage = k * (nj / H) * 128;
    for (int wide = 1; wide >= 0; --wide) {
      const int fixed = base + TC_EPI_WARPS * 2 * (wide ? TC_OUT_BUF : TC_OUT_BUF / 2);   // output staging
      int sa, sb;
      if (mt == 2) {
        int n = (TC_SMEM_LIMIT - fixed) / (a_stage + b_stage);
        if (n > 4) n = 4;
        if (n < 2) continue;
        sa = sb = n;
      } else {
        const bool few_k = C <= 640;
        sa = few_k ? 3 : 2;
        sb = few_k ? 2 : TC_SB_MAX;
        const int sb_fit = (TC_SMEM_LIMIT - fixed - sa * a_stage) / b_stage;
        if (sb > sb_fit) sb = sb_fit;
        if (sb < 2) {            // not enough room: fall back to the minimum x ring
          sa = 2;
          sb = (TC_SMEM_LIMIT - fixed - sa * a_stage) / b_stage;
          if (sb > TC_SB_MAX) sb = TC_SB_MAX;
        }
        if (sb < 2) continue;
      }
      pl.F = F; pl.P = P; pl.C = C; pl.k = k;
      pl.Cout = Cout;
      pl.NJ = nj;
      pl.MT = mt;
      pl.H = H;
      pl.b_rows = nj / H;
      pl.n_acc = n_acc;
      pl.n_slabs = Cout / nj;
      pl.slabs_per_out = cpo / nj;
      pl.n_fblk = (F + TC_M - 1) / TC_M;
      pl.sel_lo = pl.n_sel = pl.n_fblk;
      pl.sel_hi0 = 0;
      pl.n_tiles = (long long)P * pl.n_fblk;
      pl.n_jobs = ((pl.n_tiles + H * mt - 1) / (H * mt)) * pl.n_slabs;
      pl.n_cb = C / TC_KB;
      pl.n_stage = pl.n_cb;
      pl.a_rows = a_rows;
      pl.a_tile = a_tile;
      pl.a_stage = a_stage;
      pl.b_tap = (nj / H) * 128;
      pl.b_kb = k * pl.b_tap;
      pl.b_stage = b_stage;
      pl.sa = sa;
      pl.sb = sb;
      pl.hT = hT;
      pl.n_tab = n_tab;
      pl.wide = wide;
      pl.smem = fixed + sa * a_stage + sb * b_stage;
      if (pl.smem <= TC_SMEM_LIMIT) return true;
    }
  }
  return false;
}

// Tile t of a launch -> its frame block and position (the launch covers the
// plan's selected frame blocks of every position).
__device__ __forceinline__ void tc_tile_pos(const TcPlan& pl, long long t, int& fb, int& p) {
  const int s = (int)(t % pl.n_sel);
  p = (int)(t / pl.n_sel);
  fb = s < pl.sel_lo ? s : pl.sel_hi0 + (s - pl.sel_lo);
}

// The 4k MMAs of one tile and one K-block: k taps x 4 K steps of 16 channels.
// Tap t reads the x tile shifted down by t rows of 128 B (8 units of 16 B);
// K step s adds 32 B inside the swizzled x rows and two 8-column groups in w.
// KT > 0: taps known at compile time, every offset an immediate.
template <bool PAIR>
__device__ __forceinline__ void tc_umma(uint32_t d_tmem, uint64_t ad, uint64_t bd, uint32_t idesc,
                                        uint32_t acc) {
  if constexpr (PAIR) umma_bf16_pair(d_tmem, ad, bd, idesc, acc);
  else umma_bf16(d_tmem, ad, bd, idesc, acc);
}

template <int KT, bool PAIR>
__device__ __forceinline__ void tc_issue_taps(uint32_t d_tmem, uint64_t ad, uint64_t bd,
                                              uint32_t bt16, uint32_t bk16, uint32_t idesc,
                                              uint32_t acc0, int k) {
  if constexpr (KT > 0) {
#pragma unroll
    for (int t = 0; t < KT; ++t) {
#pragma unroll
      for (int s = 0; s < 4; ++s)
        tc_umma<PAIR>(d_tmem, ad + (uint64_t)(8 * t + 2 * s), bd + (uint64_t)(t * bt16 + s * bk16),
                      idesc, (t == 0 && s == 0) ? acc0 : 1u);
    }
  } else {
    for (int t = 0; t < k; ++t) {
#pragma unroll
      for (int s = 0; s < 4; ++s)
        tc_umma<PAIR>(d_tmem, ad + (uint64_t)(8 * t + 2 * s), bd + (uint64_t)(t * bt16 + s * bk16),
                      idesc, (t == 0 && s == 0) ? acc0 : 1u);
    }
  }
}

// Commit: arrive on `bar` (in both CTAs of a pair) once this thread's
// outstanding MMAs are done.
template <bool PAIR>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if constexpr (PAIR) umma_commit_pair_mc(bar, 0x3);
  else umma_commit(bar);
}

// Epilogue of one chunk of a tile row, already + bias and packed to bf16
// pairs, into the staging buffer.  w64: 64 channels (lo, hi) as a 128-byte
// row, 16-byte chunk i at i ^ (lane & 7) (128-byte swizzle); else 32
// channels (lo) as a 64-byte row, chunk i at i ^ ((lane >> 1) & 3) (64-byte
// swizzle).  Either way the eight rows a quarter-warp writes at once hit
// distinct banks.
__device__ __forceinline__ void epi_stage_chunk(uint32_t stage, int lane, const uint32_t (&lo)[16],
                                                const uint32_t (&hi)[16], bool w64) {
  if (w64) {
    const uint32_t row = stage + (uint32_t)lane * 128u, sw = (uint32_t)(lane & 7);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      sts128(row + (((uint32_t)i ^ sw) << 4),
             make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]));
#pragma unroll
    for (int i = 0; i < 4; ++i)
      sts128(row + (((uint32_t)(4 + i) ^ sw) << 4),
             make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]));
  } else {
    const uint32_t row = stage + (uint32_t)lane * 64u, sw = (uint32_t)((lane >> 1) & 3);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      sts128(row + (((uint32_t)i ^ sw) << 4),
             make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]));
  }
}

// Bounded wait; cluster-scope acquire in the pair form, where the barrier is
// signalled from the other CTA (remote arrivals, commits multicast to both).
template <bool PAIR>
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, unsigned int* err,
                                        unsigned int code) {
  if constexpr (PAIR) return mbar_wait_bounded_cluster(bar, parity, err, code);
  else return mbar_wait_bounded(bar, parity, err, code);
}

// PAIR: a cluster of two CTAs on two SMs runs tcgen05.mma.cta_group::2 with
// M = 256.  Each CTA holds its own MT tiles of x (A rows 0..127 of the MMA in
// the even CTA, 128..255 in the odd one) and HALF of every weight block (N/2
// rows each), and its own 128 accumulator lanes in TMEM.  The even CTA's
// thread issues the MMAs; both CTAs' loads complete on the even CTA's full
// barriers, the commits go to both CTAs' barriers, and the epilogues of both
// arrive on the even CTA's accumulator-empty barriers.  Per SM this halves
// the weight bytes streamed from L2 and the B operand read from shared
// memory per MMA.
template <int KT, int MT, bool PAIR>
__global__ void __launch_bounds__(TC_THREADS, 1)
    temporal_conv_tc_kernel(const __grid_constant__ TcMaps maps, const TcPlan pl,
                            const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sA = base;
  const uint32_t sB = sA + pl.sa * pl.a_stage;
  const uint32_t sOut = sB + pl.sb * pl.b_stage;       // output staging, 1024-aligned
  const uint32_t out_buf = pl.wide ? TC_OUT_BUF : TC_OUT_BUF / 2;   // bytes of one staging buffer
  const uint32_t sBar = sOut + TC_EPI_WARPS * 2 * out_buf;
  // barrier block: a_full[SA] a_empty[SA] b_full[SB] b_empty[SB] acc_full[4] acc_empty[4] drain tmem_slot
  const uint32_t a_full = sBar, a_empty = a_full + 8 * TC_SA_MAX;
  const uint32_t b_full = a_empty + 8 * TC_SA_MAX, b_empty = b_full + 8 * TC_SB_MAX;
  const uint32_t acc_full = b_empty + 8 * TC_SB_MAX, acc_empty = acc_full + 32;
  const uint32_t drain = acc_empty + 32, tmem_slot = drain + 8;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = KT > 0 ? KT : pl.k;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const long long cid = PAIR ? blockIdx.x / 2 : blockIdx.x;        // cluster (job walker) index
  const long long n_cl = PAIR ? gridDim.x / 2 : gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < pl.sa; ++i) {
      mbar_init(a_full + 8 * i, PAIR ? 2 : 1);       // one arrive.expect_tx per CTA
      mbar_init(a_empty + 8 * i, 1);
    }
    for (int i = 0; i < pl.sb; ++i) { mbar_init(b_full + 8 * i, 1); mbar_init(b_empty + 8 * i, 1); }
    for (int i = 0; i < pl.n_acc; ++i) {
      mbar_init(acc_full + 8 * i, 1);
      mbar_init(acc_empty + 8 * i, PAIR ? 2 * TC_EPI_WARPS : TC_EPI_WARPS);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
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
  if constexpr (PAIR) cluster_sync();               // both CTAs' barriers are initialised
  tc_fence_after();
  uint32_t tmem_base;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem_base) : "r"(tmem_slot));
  // The even CTA's full and accumulator-empty barriers, as cluster addresses.
  const uint32_t lead_a_full = PAIR ? mapa_shared(a_full, 0) : a_full;
  const uint32_t lead_acc_empty = PAIR ? mapa_shared(acc_empty, 0) : acc_empty;

  const int halo = k / 2;
  const int cb_rot = (int)(cid % pl.n_cb);          // the same K-block order in both CTAs
  // Two tiles per job (and every pair plan) use equal x and w rings: one
  // barrier pair per stage covers both, so a K-block costs one wait and one
  // commit.  One tile per job keeps separate rings.
  constexpr bool UNI = MT == 2;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 takes the ring waits and posts the expected bytes; the stage's
    // copies are then issued by different lanes (x box of tile m by lane m,
    // the weights by lane MT): one thread issuing every copy would serialise
    // them on its issue latency.
    int sa = 0, pa = 0, sbi = 0, pb = 0;           // ring positions as (stage, phase) counters
    bool a_used = false, b_used = false;           // first pass over a ring needs no wait
    bool ok = true;
    const uint32_t a_bytes = (uint32_t)(MT * pl.a_rows) * 128u;
    for (long long job = cid; job < pl.n_jobs && ok; job += n_cl) {
      const int slab = (int)(job % pl.n_slabs);
      const long long tile0 = (job / pl.n_slabs) * (pl.H * MT) + rank * MT;
      // Frame row and position of each tile of the job; p == P past the
      // last tile, which reads as zeros.
      int frow[MT], pos[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        int fb;
        tc_tile_pos(pl, tile0 + m, fb, pos[m]);
        frow[m] = fb * TC_M - halo + args.x_off;
      }
      // Packed weights of (slab, K-block 0): k contiguous tap blocks per K-block
      // (per CTA of a pair: its half).
      const bf16* wslab = args.wpk + (size_t)slab * pl.n_cb * (pl.b_kb / 2);
      const int wblk0 = (slab * pl.n_cb * pl.H + (int)rank) * k;   // pair: block of (slab, 0, rank, 0)
      for (int is = 0; is < pl.n_stage; ++is) {
        // Stage `is` holds K-block (is + cb_rot) mod n_cb of the job.
        const int cb = (is + cb_rot) % pl.n_cb;
        const uint32_t a_bar = PAIR ? lead_a_full + 8 * sa : a_full + 8 * sa;
        const uint32_t b_bar = UNI ? a_bar : b_full + 8 * sbi;   // shared stage: one barrier
        bool go = true;
        if (lane == 0) {
          go = !a_used || tc_wait<PAIR>(a_empty + 8 * sa, (uint32_t)(pa ^ 1), args.err,
                                        VI_DEV_ERR_TMA_TIMEOUT);
          if (go) {
            if constexpr (PAIR) mbar_arrive_expect_tx_cluster(a_bar, a_bytes + (uint32_t)pl.b_kb);
            else mbar_arrive_expect_tx(a_bar, a_bytes + (UNI ? (uint32_t)pl.b_kb : 0u));
          }
          if (go && !UNI) {
            go = !b_used || tc_wait<PAIR>(b_empty + 8 * sbi, (uint32_t)(pb ^ 1), args.err,
                                              VI_DEV_ERR_TMA_TIMEOUT);
            if (go) mbar_arrive_expect_tx(b_bar, (uint32_t)pl.b_kb);
          }
        }
        if (!__shfl_sync(0xffffffffu, go ? 1 : 0, 0)) { ok = false; break; }
        if (lane < MT) {
          // (a select, not a run-time array index, keeps frow/pos in registers)
          const uint32_t dst = sA + sa * pl.a_stage + (uint32_t)lane * pl.a_tile;
          const int fr = lane == 0 ? frow[0] : frow[MT - 1], ps = lane == 0 ? pos[0] : pos[MT - 1];
          if constexpr (PAIR) tma_load_3d_pair(dst, &maps.x, cb * TC_KB, fr, ps, a_bar);
          else tma_load_3d(dst, &maps.x, cb * TC_KB, fr, ps, a_bar);
        } else if (lane == MT) {
          if constexpr (PAIR)
            tma_load_3d_pair(sB + sbi * pl.b_stage, &maps.w, 0, 0, wblk0 + cb * pl.H * k, b_bar);
          else
            bulk_load(sB + sbi * pl.b_stage, wslab + (size_t)cb * (pl.b_kb / 2), (uint32_t)pl.b_kb,
                      b_bar);
        }
        __syncwarp();
        if (++sa == pl.sa) { sa = 0; pa ^= 1; a_used = true; }
        if (++sbi == pl.sb) { sbi = 0; pb ^= 1; b_used = true; }
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
      const uint32_t bt16 = (uint32_t)pl.b_tap >> 4;   // one tap's block in w
      const uint32_t bk16 = (2u * lbo_b) >> 4;          // one K step of 16 in w
      const uint32_t at16 = (uint32_t)pl.a_tile >> 4;   // next tile of an x stage
      int sa = 0, pa = 0, sbi = 0, pb = 0;
      // Accumulator ring: n_acc slots of NJ columns, one per tile, in order.
      int slot = 0, pslot = 0;
      bool slot_used = false;
      bool ok = true;
      for (long long job = cid; job < pl.n_jobs && ok; job += n_cl) {
        // This job's accumulator slots and the parity of their last release.
        int js[MT], jp[MT];
        bool ju[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          js[m] = slot; jp[m] = pslot; ju[m] = slot_used;
          if (++slot == pl.n_acc) { slot = 0; pslot ^= 1; slot_used = true; }
        }
        for (int is = 0; is < pl.n_stage && ok; ++is) {
          if (!tc_wait<PAIR>(a_full + 8 * sa, (uint32_t)pa, args.err, VI_DEV_ERR_TMA_TIMEOUT)) {
            ok = false;
            break;
          }
          if constexpr (!UNI) {
            if (!tc_wait<PAIR>(b_full + 8 * sbi, (uint32_t)pb, args.err, VI_DEV_ERR_TMA_TIMEOUT)) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint64_t ad_stage = ad_base + (uint64_t)(sa * a_st16);
          const uint64_t bd_stage = bd_base + (uint64_t)((UNI ? sa : sbi) * b_st16);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (is == 0) {
              // The slot must have been drained by the epilogue of its last tile.
              if (ju[m] && !tc_wait<PAIR>(acc_empty + 8 * js[m], (uint32_t)(jp[m] ^ 1), args.err,
                                          VI_DEV_ERR_MMA_TIMEOUT)) { ok = false; break; }
              tc_fence_after();
            }
            tc_issue_taps<KT, PAIR>(tmem_base + (uint32_t)(js[m] * pl.NJ),
                                    ad_stage + (uint64_t)(m * at16), bd_stage, bt16, bk16, idesc,
                                    is > 0 ? 1u : 0u, k);
            if (is == pl.n_stage - 1) tc_commit<PAIR>(acc_full + 8 * js[m]);   // accumulator ready
          }
          if (!ok) break;
          if constexpr (!UNI) tc_commit<PAIR>(b_empty + 8 * sbi);   // frees the w stage
          tc_commit<PAIR>(a_empty + 8 * sa);   // frees the x stage (and the w stage if shared)
          if (++sa == pl.sa) { sa = 0; pa ^= 1; }
          if constexpr (!UNI) {
            if (++sbi == pl.sb) { sbi = 0; pb ^= 1; }
          }
        }
      }
      // Every MMA this thread issued must finish before TMEM is released.
      tc_commit<PAIR>(drain);
      tc_wait<PAIR>(drain, 0, args.err, VI_DEV_ERR_MMA_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp q owns TMEM lanes 32q .. 32q+31 (frames 32q .. of the tile) and
    // writes them on its own: no barrier across the four warps, and each
    // warp's lane 0 issues its own TMA stores (four store streams).  A chunk
    // is 64 channels where the plan has room for the staging (32 for the
    // last chunk of a slab of 32 mod 64 channels), else 32.
    const int q = warp & 3;
    const uint32_t my_out = sOut + (uint32_t)q * 2u * out_buf;   // two staging buffers
    int ob = 0;                                  // staging buffer of the next chunk
    int buf = 0, pacc = 0;                       // accumulator ring, as the MMA issuer walks it
    bool ok = true;
    for (long long job = cid; job < pl.n_jobs && ok; job += n_cl) {
      const int slab = (int)(job % pl.n_slabs);
      const int out = slab / pl.slabs_per_out;                 // output tensor of this slab
      const int ch0 = (slab - out * pl.slabs_per_out) * pl.NJ; // its first channel there
      for (int mt = 0; mt < MT; ++mt) {
        // The lanes take the (bounded) wait's outcome together.
        const bool got = __all_sync(0xffffffffu, tc_wait<PAIR>(acc_full + 8 * buf, (uint32_t)pacc,
                                                                args.err, VI_DEV_ERR_MMA_TIMEOUT));
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        const long long tile = (job / pl.n_slabs) * (pl.H * MT) + rank * MT + mt;
        int fb, p;
        tc_tile_pos(pl, tile, fb, p);
        const bool tile_ok = tile < pl.n_tiles;
        // This row's bias table: by its distance to each video end, capped at
        // hT (one table, the plain bias, when hT == 0).
        const int f = fb * TC_M + 32 * q + lane;
        const int lo = min(f, pl.hT), hi = max(min(pl.F - 1 - f, pl.hT), 0);
        // (read through L1: every warp of every CTA reads the same few KB)
        const float* bs = args.btab + (lo * (pl.hT + 1) + hi) * pl.Cout + slab * pl.NJ;
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * pl.NJ);
        // The tile row group by group (32 columns): TMEM -> registers, + bias,
        // -> bf16 pairs (16 registers a group, so that the whole row fits
        // beside the other roles' state).  The accumulator goes back to the
        // MMA after the last group; the staging and stores of the tile
        // overlap the next tiles' MMAs.  Loops unrolled: registers indexed at
        // compile time only.
        uint32_t pk[TC_NJ_MAX / 32][16];
#pragma unroll
        for (int g = 0; g < TC_NJ_MAX / 32; ++g) {
          if (32 * g >= pl.NJ) break;
          uint32_t r[32];
          tmem_ld32(taddr + 32u * g, r);
          // (the bias tables are 128-byte aligned per 32 channels; read
          // through L1: every warp of every CTA reads the same few KB)
          const float4* b4 = reinterpret_cast<const float4*>(bs + 32 * g);
          float4 bv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) bv[i] = __ldg(b4 + i);
          tmem_wait_ld_dep(r);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            pk[g][2 * i] = pack2_bf16(__uint_as_float(r[4 * i]) + bv[i].x,
                                      __uint_as_float(r[4 * i + 1]) + bv[i].y);
            pk[g][2 * i + 1] = pack2_bf16(__uint_as_float(r[4 * i + 2]) + bv[i].z,
                                          __uint_as_float(r[4 * i + 3]) + bv[i].w);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(lead_acc_empty + 8 * buf);
          else mbar_arrive(acc_empty + 8 * buf);
        }
        // Chunks: 64 channels (groups g, g+1) where the plan is wide and
        // they fit, else 32 (group g).  Loops unrolled: registers indexed
        // at compile time only.
        bool taken = false;                   // group g went out with group g-1
#pragma unroll
        for (int g = 0; g < TC_NJ_MAX / 32; ++g) {
          if (32 * g >= pl.NJ) break;
          if (taken) { taken = false; continue; }
          const bool w64 = g + 1 < TC_NJ_MAX / 32 && pl.wide && 32 * g + 64 <= pl.NJ;
          const uint32_t stage = my_out + (uint32_t)ob * out_buf;
          if (lane == 0) bulk_wait_read_le1();   // the store that last read this buffer is done
          __syncwarp();
          if (tile_ok)
            epi_stage_chunk(stage, lane, pk[g], pk[g + 1 < TC_NJ_MAX / 32 ? g + 1 : g], w64);
          fence_proxy_async_smem();           // the writes are visible to the TMA store
          __syncwarp();
          if (lane == 0 && tile_ok) {
            // Rows past the last frame fall outside the tensor map and are dropped.
            tma_store_3d(w64 ? &maps.y[out] : &maps.y32[out], stage, ch0 + 32 * g,
                         fb * TC_M + 32 * q, p);
            bulk_commit();
          }
          ob ^= 1;
          taken = w64;
        }
        if (++buf == pl.n_acc) { buf = 0; pacc ^= 1; }
      }
    }
    if (lane == 0) bulk_wait_all();              // every output chunk has reached global memory
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

// w [C_out][C_in][k] -> [slab][cb][h][t][8 columns][NJ/H][8]: for each (slab,
// K-block, CTA h of a pair (H = 2) or h = 0 (H = 1), tap) an NJ/H x 64 K-major
// block in the no-swizzle layout, the k tap blocks of a (slab, K-block, h)
// contiguous.  coef != null (GroupNorm folded
// into the conv): each input channel's weights are scaled by its GroupNorm
// factor a_ci first, W'[co][ci][t] = bf16(w[co][ci][t] * a_ci), and the bias
// tables come from temporal_conv_fold_bias; otherwise this kernel also
// writes the one bias table, b in fp32.
__device__ __forceinline__ bf16 tc_folded_w(const bf16* w, const float* coef, int co, int ci,
                                            int t, int C, int k) {
  const bf16 v = w[((size_t)co * C + ci) * k + t];
  return coef ? __float2bfloat16_rn(__bfloat162float(v) * coef[4 * ci + 1]) : v;
}

__global__ void temporal_conv_pack_w(const bf16* __restrict__ w, const float* __restrict__ coef,
                                     bf16* __restrict__ wpk, const bf16* __restrict__ b,
                                     float* __restrict__ tab, int C, int Cout, int k, int NJ,
                                     int H) {
  const long long total = (long long)Cout * C * k;
  // Plain conv (no GroupNorm folded in): its one bias table is b in fp32.
  if (!coef)
    for (int co = blockIdx.x * blockDim.x + threadIdx.x; co < Cout; co += gridDim.x * blockDim.x)
      tab[co] = __bfloat162float(b[co]);
  const int n_cb = C / TC_KB;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int R = NJ / H;
    const int e = (int)(i & 7);
    long long r = i >> 3;
    const int n = (int)(r % R); r /= R;
    const int col = (int)(r % 8); r /= 8;
    const int t = (int)(r % k); r /= k;
    const int h = (int)(r % H); r /= H;
    const int cb = (int)(r % n_cb);
    const int slab = (int)(r / n_cb);
    wpk[i] = tc_folded_w(w, coef, slab * NJ + h * R + n, cb * TC_KB + col * 8 + e, t, C, k);
  }
}

// Bias tables of the GroupNorm-folded conv.  With x_n = (x - m) a + beta on
// the frames of the video and 0 outside, the conv of x_n is, per output
// channel co and frame f,
//   b[co] + sum_t sum_ci W[co,ci,t] x_n[f+t-h, ci]
//     = acc + b[co] + sum_{t valid} sum_ci (W[co,ci,t] beta_ci - W'[co,ci,t] m_ci)
// where acc = sum_t sum_ci W'[co,ci,t] x[f+t-h, ci] is what the tensor cores
// compute from the raw x (zero outside the video) and W' = bf16(W a) are the
// folded weights.  The mean term uses the same rounded W' as acc, so the
// means cancel exactly and the rounding of W' only scales x - m.  A tap t is
// valid when frame f+t-h lies in the video: with lo = min(f, h) frames
// before f and hi = min(F-1-f, h) after it, t in [h - lo, h + hi].  One
// block per output channel; table (lo, hi) at [(lo (h+1) + hi) Cout + co].
__global__ void __launch_bounds__(128) temporal_conv_fold_bias(
    const bf16* __restrict__ w, const bf16* __restrict__ b, const float* __restrict__ coef,
    float* __restrict__ tab, int C, int Cout, int k) {
  constexpr int MAXK = 8;
  __shared__ double part[MAXK][4];
  const int co = blockIdx.x, h = k / 2;
  double acc[MAXK];
  for (int t = 0; t < k; ++t) acc[t] = 0.0;
  for (int ci = threadIdx.x; ci < C; ci += blockDim.x) {
    const double m = coef[4 * ci], beta = coef[4 * ci + 2];
    for (int t = 0; t < k; ++t) {
      const double wv = __bfloat162float(w[((size_t)co * C + ci) * k + t]);
      const double wf = __bfloat162float(tc_folded_w(w, coef, co, ci, t, C, k));
      acc[t] += wv * beta - wf * m;
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = 0; t < k; ++t) {
    double v = acc[t];
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) part[t][warp] = v;
  }
  __syncthreads();
  if (threadIdx.x < (h + 1) * (h + 1)) {
    const int lo = threadIdx.x / (h + 1), hi = threadIdx.x % (h + 1);
    double sum = __bfloat162float(b[co]);
    for (int t = h - lo; t <= h + hi; ++t)
      sum += part[t][0] + part[t][1] + part[t][2] + part[t][3];
    tab[(size_t)threadIdx.x * Cout + co] = (float)sum;
  }
}

bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                 CUtensorMapDataType dt);

// Tiles per job of the default plan (2: every weight stage feeds two tiles).
constexpr int TC_MT_DEFAULT = 2;
// The default plan runs on a CTA pair for convs of k >= 3 taps with at least
// this many K-blocks per job, where the pair plan keeps the slab width.
// Measured on B200 (cycles per 128-row MMA per SM, as dispatched): C = 640,
// 10 K-blocks: 95 on a pair against 99 on one SM; C = 320, 5 K-blocks: 108
// against 103 (the pair's accumulator hand-off, which waits for both CTAs'
// epilogues, costs more per job than the pair saves); the single-tap GEMMs of
// the attention module ran slower on pairs as well.
constexpr int TC_PAIR_MIN_KBLOCKS = 10;
// Largest tap count of the GroupNorm-folded conv (bias tables per distance to
// the video ends: (k/2 + 1)^2 of them).
constexpr int TC_FOLD_MAX_K = 7;

bool temporal_conv_tc_ok(int F, int P, int C, int k) {
  TcPlan pl;
  return F > 0 && P > 0 && tc_plan(F, P, C, C, 1, k, pl, 0, 1);
}

bool temporal_conv_tc_norm_ok(int F, int P, int C, int k) {
  TcPlan pl;
  return F > 0 && P > 0 && k <= TC_FOLD_MAX_K && tc_plan(F, P, C, C, 1, k, pl, k / 2, 1);
}

bool linear_tc_ok(int F, int P, int C, int Cout, int n_out) {
  TcPlan pl;
  return F > 0 && P > 0 && tc_plan(F, P, C, Cout, n_out, 1, pl, 0, 1);
}

template <int KT, int MT, bool PAIR>
static int tc_launch(const TcMaps& maps, const TcPlan& pl, const TcArgs& a, cudaStream_t stream) {
  static std::mutex mu;
  static bool attr_done[64] = {false};
  int dev = 0;
  VI_CUDA_TRY(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return VI_ERR_CUDA;
    if (!attr_done[dev]) {
      VI_CUDA_TRY(cudaFuncSetAttribute(temporal_conv_tc_kernel<KT, MT, PAIR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TC_SMEM_LIMIT));
      attr_done[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(TC_THREADS);
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
    if (cudaOccupancyMaxActiveClusters(&clusters, temporal_conv_tc_kernel<KT, MT, PAIR>, &cfg) !=
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
  VI_CUDA_TRY(cudaLaunchKernelEx(&cfg, temporal_conv_tc_kernel<KT, MT, PAIR>, maps, pl, a));
  note_launch();
  return VI_OK;
}

// The kernel form of a plan: taps 3 and 1 are compiled with their loops
// unrolled, any other odd k runs the tap loop at run time.
static int tc_dispatch(const TcMaps& maps, const TcPlan& pl, const TcArgs& a,
                       cudaStream_t stream) {
  const int kt = pl.k == 3 ? 3 : pl.k == 1 ? 1 : 0;
  if (pl.H == 2) {                          // CTA pair, two tiles per CTA
    switch (kt) {
      case 3: return tc_launch<3, 2, true>(maps, pl, a, stream);
      case 1: return tc_launch<1, 2, true>(maps, pl, a, stream);
      default: return tc_launch<0, 2, true>(maps, pl, a, stream);
    }
  }
  switch (kt * 10 + pl.MT) {
    case 32: return tc_launch<3, 2, false>(maps, pl, a, stream);
    case 31: return tc_launch<3, 1, false>(maps, pl, a, stream);
    case 12: return tc_launch<1, 2, false>(maps, pl, a, stream);
    case 11: return tc_launch<1, 1, false>(maps, pl, a, stream);
    case 2: return tc_launch<0, 2, false>(maps, pl, a, stream);
    default: return tc_launch<0, 1, false>(maps, pl, a, stream);
  }
}

// One call: x [P][x_rows][C] (output frame f reads x row f + x_off + t - k/2),
// w [Cout][C][k], b [Cout], outputs ys[0..n_out) each [P][F][Cout/n_out].
// coef != nullptr: the conv of the GroupNorm of x, with the GroupNorm's
// per-channel coefficients (m_c, a_c, beta_c) folded into the weights and the
// bias tables (fused GroupNorm -> conv; see temporal_conv_fold_bias).
// mt: tiles per job, 0 = the default plan (two tiles on one SM where that
// keeps the slab width, else one; a CTA pair with two tiles per CTA for
// k >= 3 convs with long jobs); 1 or 2 force that one-SM form, 4 the pair.
static int tc_run(const bf16* x, int x_rows, int x_off, const bf16* w, const bf16* b,
                  bf16* const* ys, int n_out, int F, int P, int C, int Cout, int k,
                  cudaStream_t stream, const float* coef, int mt, int part = VI_PART_ALL) {
  TcPlan pl;
  const bool fold = coef != nullptr;
  if (fold && k > TC_FOLD_MAX_K) return VI_ERR_UNSUPPORTED;
  const int hT = fold ? k / 2 : 0;
  if (mt != 0) {
    if (!tc_plan(F, P, C, Cout, n_out, k, pl, hT, mt == 4 ? 2 : mt, mt == 4))
      return VI_ERR_UNSUPPORTED;
  } else {
    if (!tc_plan(F, P, C, Cout, n_out, k, pl, hT, 1)) return VI_ERR_UNSUPPORTED;
    // Two tiles per job when that plan keeps the slab width (a narrower MMA
    // N costs more than the weight traffic it saves); on a CTA pair when that
    // keeps it too and the job is long enough to pay for the pair hand-off.
    TcPlan pl2;
    if (tc_plan(F, P, C, Cout, n_out, k, pl2, hT, TC_MT_DEFAULT) && pl2.NJ >= pl.NJ) pl = pl2;
    if (k >= 3 && C / TC_KB >= TC_PAIR_MIN_KBLOCKS &&
        tc_plan(F, P, C, Cout, n_out, k, pl2, hT, TC_MT_DEFAULT, true) && pl2.NJ >= pl.NJ)
      pl = pl2;
  }
  if (part != VI_PART_ALL) {
    // Frame blocks whose x rows (with the k/2 rows on each side) lie inside
    // the shard are interior: [a, b).  The others are the boundary blocks.
    const int h = k / 2;
    const int a = pl.n_fblk < 1 ? pl.n_fblk : 1;
    int b = (F - h) / TC_M;
    if (b > pl.n_fblk) b = pl.n_fblk;
    if (b < a) b = a;
    if (part == VI_PART_INTERIOR) {
      pl.sel_lo = 0; pl.sel_hi0 = a; pl.n_sel = b - a;
    } else {
      pl.sel_lo = a; pl.sel_hi0 = b; pl.n_sel = a + (pl.n_fblk - b);
    }
    pl.n_tiles = (long long)P * pl.n_sel;
    pl.n_jobs = ((pl.n_tiles + pl.MT - 1) / pl.MT) * pl.n_slabs;
    if (pl.n_sel == 0) return VI_OK;          // nothing in this part
  }
  unsigned int* err = device_error_word();
  if (!err) return VI_ERR_CUDA;
  TcMaps maps;
  const int cpo = Cout / n_out;
  for (int i = 0; i < n_out; ++i) {
    // y as [P][F][Cout/n_out]: boxes of 64 channels (128B swizzle) and of 32
    // channels (64B swizzle) x 32 frames x 1 position.
    const uint64_t dims[3] = {(uint64_t)cpo, (uint64_t)F, (uint64_t)P};
    const uint64_t strides[2] = {(uint64_t)cpo * 2, (uint64_t)F * cpo * 2};
    const uint32_t box64[3] = {64, 32, 1}, box32[3] = {32, 32, 1};
    if (!encode_tmap(&maps.y[i], ys[i], 3, dims, strides, box64, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
        !encode_tmap(&maps.y32[i], ys[i], 3, dims, strides, box32, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      return VI_ERR_CUDA;
  }
  for (int i = n_out; i < TC_MAX_OUT; ++i) {
    maps.y[i] = maps.y[0];
    maps.y32[i] = maps.y32[0];
  }
  {
    // x as [P][x_rows][C]: box of 64 channels x a_rows frames x 1 position, 128B swizzle.
    const uint64_t dims[3] = {(uint64_t)C, (uint64_t)x_rows, (uint64_t)P};
    const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)x_rows * C * 2};
    const uint32_t box[3] = {(uint32_t)TC_KB, (uint32_t)pl.a_rows, 1};
    if (!encode_tmap(&maps.x, x, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      return VI_ERR_CUDA;
  }
  // Scratch: the packed weights, then the bias tables (fp32).
  const size_t wbytes = (((size_t)Cout * C * k * sizeof(bf16)) + 255) / 256 * 256;
  const size_t tbytes = (size_t)pl.n_tab * Cout * sizeof(float);
  void* scratch = nullptr;
  VI_CUDA_TRY(scratch_alloc(&scratch, wbytes + tbytes, stream));
  bf16* wpk = static_cast<bf16*>(scratch);
  float* tab = reinterpret_cast<float*>(static_cast<char*>(scratch) + wbytes);
  int st = VI_OK;
  {
    const long long total = (long long)Cout * C * k;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
    temporal_conv_pack_w<<<blocks, 256, 0, stream>>>(w, coef, wpk, b, tab, C, Cout, k, pl.NJ,
                                                     pl.H);
    if (cudaGetLastError() != cudaSuccess) st = VI_ERR_CUDA; else note_launch();
  }
  if (st == VI_OK && fold) {
    temporal_conv_fold_bias<<<Cout, 128, 0, stream>>>(w, b, coef, tab, C, Cout, k);
    if (cudaGetLastError() != cudaSuccess) st = VI_ERR_CUDA; else note_launch();
  }
  if (st == VI_OK && pl.H == 2) {
    // Packed weights as blocks of b_rows rows of 128 bytes: one box = the k
    // tap blocks of one CTA's half of a (slab, K-block).
    const uint64_t dims[3] = {64, (uint64_t)pl.b_rows, (uint64_t)Cout * C * k / (64ull * pl.b_rows)};
    const uint64_t strides[2] = {128, (uint64_t)pl.b_rows * 128};
    const uint32_t box[3] = {64, (uint32_t)pl.b_rows, (uint32_t)k};
    if (!encode_tmap(&maps.w, wpk, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
      st = VI_ERR_CUDA;
  } else {
    maps.w = maps.x;                          // not read by the one-SM form
  }
  if (st == VI_OK) {
    const TcArgs a{tab, wpk, err, x_off};
    st = tc_dispatch(maps, pl, a, stream);
  }
  if (scratch_free(scratch, stream) != cudaSuccess && st == VI_OK) st = VI_ERR_CUDA;
  return st;
}

// mt: 0 for the default plan; 1 or 2 tiles per job on one SM, or 4 (a CTA
// pair, two tiles per CTA) force that job form (the tests use it to reach
// every form).
int temporal_conv_bf16_tc(const bf16* x, const bf16* w, const bf16* b, bf16* y, int F, int P,
                          int C, int k, cudaStream_t stream, const float* coef, int mt) {
  if (mt != 0 && mt != 1 && mt != 2 && mt != 4) return VI_ERR_INVALID_ARG;
  bf16* ys[1] = {y};
  return tc_run(x, F, 0, w, b, ys, 1, F, P, C, C, k, stream, coef, mt);
}

// Per-frame linear layer x [P][F][C] -> n_out tensors [P][F][Cout/n_out]
// (w [Cout][C], b [Cout]): the q/k/v projection as one GEMM of N = Cout.
int linear_bf16_tc(const bf16* x, const bf16* w, const bf16* b, bf16* const* ys, int n_out,
                   int F, int P, int C, int Cout, cudaStream_t stream) {
  return tc_run(x, F, 0, w, b, ys, n_out, F, P, C, Cout, 1, stream, nullptr, 0);
}

// One shard of a video cut along frames: x_ext [P][F_loc + 2(k/2)][C] holds
// the k/2 frames before the shard (zeros at the start of the video), the
// shard's frames and the k/2 frames after it (zeros at the end); y is
// [P][F_loc][C].  part: every frame block, only those that read no halo row
// (interior), or only the others (boundary).
int temporal_conv_bf16_tc_shard(const bf16* x_ext, const bf16* w, const bf16* b, bf16* y,
                                int F_loc, int P, int C, int k, int part, cudaStream_t stream) {
  bf16* ys[1] = {y};
  return tc_run(x_ext, F_loc + 2 * (k / 2), k / 2, w, b, ys, 1, F_loc, P, C, C, k, stream, nullptr,
                0, part);
}

}  // namespace vi
