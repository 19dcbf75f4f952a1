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
// Job = (position p, 128-frame block, slab of NJ output channels).  Per job
// the CTA runs C/64 K-blocks; each K-block stages, with TMA, the x rows
// [f0 - k/2, f0 + 128 + k/2) x 64 channels ONCE (a_rows = 127 + k rows) in the
// no-swizzle K-major layout (rows 16 bytes apart inside each 8-channel
// column, columns a_col >= 16*a_rows bytes apart, a multiple of 128), so the
// k taps read the same shared tile through descriptors whose start differs by
// 16 bytes per tap: the tap shift costs no extra load.  The
// frame coordinate -1 (and F) reads as zero from TMA's out-of-bounds fill,
// which is exactly the zero padding at the two ends of the video.  The
// k weight slabs (NJ x 64 each) come from a repacked copy of w by 1-D bulk
// copies.  One thread issues tcgen05.mma (M = 128, N = NJ, K = 16) into one
// of two TMEM accumulators; four epilogue warps drain the other one (TMEM ->
// registers, + bias, -> bf16 -> global), so the epilogue overlaps the next
// job's MMAs.
//
// Warp roles (192 threads, one CTA per SM, persistent over jobs):
//   warp 0      TMA producer (one elected thread)
//   warp 1      TMEM allocator + MMA issuer (one elected thread)
//   warps 2..5  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31
#include <mutex>

#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

constexpr int TC_M = 128;        // frames per job = UMMA M = TMEM lanes
constexpr int TC_KB = 64;        // input channels per K-block (8 columns of 8)
constexpr int TC_SA = 3;         // A (x) stages
constexpr int TC_SB_MAX = 8;     // B (w) stages at most
constexpr int TC_THREADS = 192;
constexpr int TC_TMEM_COLS = 512;
constexpr int TC_SMEM_LIMIT = 232448;   // 227 KB opt-in per CTA

struct TcPlan {
  int F, P, C, k;
  int NJ;                // output channels per job (UMMA N), multiple of 32
  int n_slabs;           // C / NJ
  int n_fblk;            // ceil(F / 128)
  long long n_jobs;      // P * n_fblk * n_slabs
  int n_cb;              // C / 64
  int a_rows;            // 127 + k
  int a_col;             // bytes between 8-channel columns of an A stage (128-aligned)
  int a_stage;           // bytes per A stage, 1024-aligned
  int b_stage;           // bytes per B stage = NJ * 64 * 2
  int sb;                // B stages
  int smem;              // dynamic shared memory bytes
};

struct TcArgs {
  const bf16* wpk;       // packed weights [slab][cb][t][8 columns][NJ][8]
  const bf16* bias;
  bf16* y;
  unsigned int* err;
};

static bool tc_plan(int F, int P, int C, int k, TcPlan& pl) {
  if (k < 1 || k % 2 == 0 || 127 + k > 256 || C % TC_KB != 0) return false;
  int nj = 0;
  for (int cand = 256; cand >= 32; cand -= 32)
    if (C % cand == 0) { nj = cand; break; }
  if (nj == 0) return false;
  pl.F = F; pl.P = P; pl.C = C; pl.k = k;
  pl.NJ = nj;
  pl.n_slabs = C / nj;
  pl.n_fblk = (F + TC_M - 1) / TC_M;
  pl.n_jobs = (long long)P * pl.n_fblk * pl.n_slabs;
  pl.n_cb = C / TC_KB;
  pl.a_rows = 127 + k;
  pl.a_col = ((pl.a_rows * 16 + 127) / 128) * 128;     // TMA destinations are 128B-aligned
  pl.a_stage = ((8 * pl.a_col + 1023) / 1024) * 1024;
  pl.b_stage = nj * TC_KB * 2;
  const int fixed = 1024 /* align slack */ + TC_SA * pl.a_stage + 4 * C /* bias */ + 512 /* bars */;
  int sb = (TC_SMEM_LIMIT - fixed) / pl.b_stage;
  if (sb > TC_SB_MAX) sb = TC_SB_MAX;
  if (sb < 2) return false;
  pl.sb = sb;
  pl.smem = fixed + sb * pl.b_stage;
  return pl.smem <= TC_SMEM_LIMIT;
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    temporal_conv_tc_kernel(const __grid_constant__ CUtensorMap tmx, const TcPlan pl,
                            const TcArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sA = base;
  const uint32_t sB = sA + TC_SA * pl.a_stage;
  const uint32_t sBias = sB + pl.sb * pl.b_stage;
  const uint32_t sBar = sBias + ((4 * pl.C + 63) / 64) * 64;
  // barrier block: a_full[SA] a_empty[SA] b_full[SB] b_empty[SB] acc_full[2] acc_empty[2] drain tmem_slot
  const uint32_t a_full = sBar, a_empty = a_full + 8 * TC_SA;
  const uint32_t b_full = a_empty + 8 * TC_SA, b_empty = b_full + 8 * TC_SB_MAX;
  const uint32_t acc_full = b_empty + 8 * TC_SB_MAX, acc_empty = acc_full + 16;
  const uint32_t drain = acc_empty + 16, tmem_slot = drain + 8;
  float* bias_s = reinterpret_cast<float*>(smem_raw + (sBias - smem_u32(smem_raw)));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < TC_SA; ++i) { mbar_init(a_full + 8 * i, 1); mbar_init(a_empty + 8 * i, 1); }
    for (int i = 0; i < pl.sb; ++i) { mbar_init(b_full + 8 * i, 1); mbar_init(b_empty + 8 * i, 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(acc_full + 8 * i, 1); mbar_init(acc_empty + 8 * i, 4); }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  for (int c = threadIdx.x; c < pl.C; c += blockDim.x) bias_s[c] = to_f32(args.bias[c]);
  if (warp == 1) {
    tmem_alloc(tmem_slot, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t tmem_base;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem_base) : "r"(tmem_slot));

  const int halo = pl.k / 2;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      long long a_it = 0, b_it = 0;
      bool ok = true;
      for (long long job = blockIdx.x; job < pl.n_jobs && ok; job += gridDim.x) {
        const int slab = (int)(job % pl.n_slabs);
        const long long rest = job / pl.n_slabs;
        const int fb = (int)(rest % pl.n_fblk);
        const int p = (int)(rest / pl.n_fblk);
        const int f0 = fb * TC_M;
        for (int cb = 0; cb < pl.n_cb && ok; ++cb) {
          const int sa = (int)(a_it % TC_SA);
          const long long ua = a_it / TC_SA;
          if (ua > 0 && !mbar_wait_bounded(a_empty + 8 * sa, (uint32_t)((ua - 1) & 1), args.err,
                                           VI_DEV_ERR_TMA_TIMEOUT)) { ok = false; break; }
          const uint32_t dst = sA + sa * pl.a_stage;
          mbar_arrive_expect_tx(a_full + 8 * sa, (uint32_t)pl.a_rows * 128u);
          // 8 columns of 8 channels; column c lands at dst + c * a_col.
#pragma unroll 1
          for (int c = 0; c < 8; ++c)
            tma_load_3d(dst + c * pl.a_col, &tmx, cb * TC_KB + c * 8, f0 - halo, p,
                        a_full + 8 * sa);
          ++a_it;
          for (int t = 0; t < pl.k; ++t) {
            const int s = (int)(b_it % pl.sb);
            const long long ub = b_it / pl.sb;
            if (ub > 0 && !mbar_wait_bounded(b_empty + 8 * s, (uint32_t)((ub - 1) & 1), args.err,
                                             VI_DEV_ERR_TMA_TIMEOUT)) { ok = false; break; }
            mbar_arrive_expect_tx(b_full + 8 * s, (uint32_t)pl.b_stage);
            const bf16* src = args.wpk + ((size_t)(slab * pl.n_cb + cb) * pl.k + t) *
                                             (size_t)(pl.NJ * TC_KB);
            bulk_load(sB + s * pl.b_stage, src, (uint32_t)pl.b_stage, b_full + 8 * s);
            ++b_it;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(TC_M, pl.NJ);
      const uint32_t lbo_a = (uint32_t)pl.a_col, lbo_b = (uint32_t)pl.NJ * 16u;
      long long a_it = 0, b_it = 0, j_it = 0;
      bool ok = true;
      for (long long job = blockIdx.x; job < pl.n_jobs && ok; job += gridDim.x, ++j_it) {
        const int buf = (int)(j_it & 1);
        const long long use = j_it >> 1;
        if (use > 0 && !mbar_wait_bounded(acc_empty + 8 * buf, (uint32_t)((use - 1) & 1), args.err,
                                          VI_DEV_ERR_MMA_TIMEOUT)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * pl.NJ);
        for (int cb = 0; cb < pl.n_cb && ok; ++cb) {
          const int sa = (int)(a_it % TC_SA);
          if (!mbar_wait_bounded(a_full + 8 * sa, (uint32_t)((a_it / TC_SA) & 1), args.err,
                                 VI_DEV_ERR_TMA_TIMEOUT)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = sA + sa * pl.a_stage;
          for (int t = 0; t < pl.k; ++t) {
            const int s = (int)(b_it % pl.sb);
            if (!mbar_wait_bounded(b_full + 8 * s, (uint32_t)((b_it / pl.sb) & 1), args.err,
                                   VI_DEV_ERR_TMA_TIMEOUT)) { ok = false; break; }
            tc_fence_after();
            const uint32_t b_base = sB + s * pl.b_stage;
#pragma unroll
            for (int ks = 0; ks < TC_KB / 16; ++ks) {
              const uint64_t ad =
                  umma_desc_kmajor_noswizzle(a_base + 16u * t + 2u * ks * lbo_a, lbo_a, 128u);
              const uint64_t bd =
                  umma_desc_kmajor_noswizzle(b_base + 2u * ks * lbo_b, lbo_b, 128u);
              umma_bf16(d_tmem, ad, bd, idesc, (cb | t | ks) != 0 ? 1u : 0u);
            }
            umma_commit(b_empty + 8 * s);       // frees the w stage when these MMAs finish
            ++b_it;
          }
          umma_commit(a_empty + 8 * sa);        // frees the x stage
          ++a_it;
        }
        umma_commit(acc_full + 8 * buf);        // accumulator ready for the epilogue
      }
      // Wait for every MMA this thread issued before TMEM can be released.
      umma_commit(drain);
      mbar_wait_bounded(drain, 0, args.err, VI_DEV_ERR_MMA_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                      // TMEM lane quadrant of this warp
    const int m = 32 * q + lane;                 // frame within the job
    long long j_it = 0;
    for (long long job = blockIdx.x; job < pl.n_jobs; job += gridDim.x, ++j_it) {
      const int buf = (int)(j_it & 1);
      if (!mbar_wait_bounded(acc_full + 8 * buf, (uint32_t)((j_it >> 1) & 1), args.err,
                             VI_DEV_ERR_MMA_TIMEOUT))
        break;
      tc_fence_after();
      const int slab = (int)(job % pl.n_slabs);
      const long long rest = job / pl.n_slabs;
      const int fb = (int)(rest % pl.n_fblk);
      const long long p = rest / pl.n_fblk;
      const int f = fb * TC_M + m;
      const bool valid = f < pl.F;
      bf16* out = args.y + ((size_t)p * pl.F + (valid ? f : 0)) * pl.C + (size_t)slab * pl.NJ;
      const float* bs = bias_s + slab * pl.NJ;
      for (int c0 = 0; c0 < pl.NJ; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * pl.NJ + c0), r);
        tmem_wait_ld();
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2_bf16(__uint_as_float(r[2 * i]) + bs[c0 + 2 * i],
                               __uint_as_float(r[2 * i + 1]) + bs[c0 + 2 * i + 1]);
          uint4* o = reinterpret_cast<uint4*>(out + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + 8 * buf);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

// w [C_out][C_in][k] -> [slab][cb][t][8 columns][NJ][8]: for each (slab, K-block,
// tap) an NJ x 64 K-major tile in the no-swizzle layout, contiguous.
__global__ void temporal_conv_pack_w(const bf16* __restrict__ w, bf16* __restrict__ wpk, int C,
                                     int k, int NJ) {
  const long long total = (long long)C * C * k;
  const int n_cb = C / TC_KB;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int e = (int)(i & 7);
    long long r = i >> 3;
    const int n = (int)(r % NJ); r /= NJ;
    const int col = (int)(r % 8); r /= 8;
    const int t = (int)(r % k); r /= k;
    const int cb = (int)(r % n_cb);
    const int slab = (int)(r / n_cb);
    const int co = slab * NJ + n, ci = cb * TC_KB + col * 8 + e;
    wpk[i] = w[((size_t)co * C + ci) * k + t];
  }
}

bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                 CUtensorMapDataType dt);

bool temporal_conv_tc_ok(int F, int P, int C, int k) {
  TcPlan pl;
  return F > 0 && P > 0 && tc_plan(F, P, C, k, pl);
}

int temporal_conv_bf16_tc(const bf16* x, const bf16* w, const bf16* b, bf16* y, int F, int P,
                          int C, int k, cudaStream_t stream) {
  TcPlan pl;
  if (!tc_plan(F, P, C, k, pl)) return VI_ERR_UNSUPPORTED;
  unsigned int* err = device_error_word();
  if (!err) return VI_ERR_CUDA;
  // x as [P][F][C]: box of 8 channels x a_rows frames x 1 position, no swizzle.
  CUtensorMap tmx;
  const uint64_t dims[3] = {(uint64_t)C, (uint64_t)F, (uint64_t)P};
  const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)F * C * 2};
  const uint32_t box[3] = {8, (uint32_t)pl.a_rows, 1};
  if (!encode_tmap(&tmx, x, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
    return VI_ERR_CUDA;

  static std::mutex mu;
  static bool attr_done[64] = {false};
  int dev = 0;
  VI_CUDA_TRY(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64 && !attr_done[dev]) {
      VI_CUDA_TRY(cudaFuncSetAttribute(temporal_conv_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TC_SMEM_LIMIT));
      attr_done[dev] = true;
    }
  }
  const size_t wbytes = (size_t)C * C * k * sizeof(bf16);
  void* wpk = nullptr;
  VI_CUDA_TRY(cudaMallocAsync(&wpk, wbytes, stream));
  int st = VI_OK;
  {
    const long long total = (long long)C * C * k;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
    temporal_conv_pack_w<<<blocks, 256, 0, stream>>>(w, static_cast<bf16*>(wpk), C, k, pl.NJ);
    if (cudaGetLastError() != cudaSuccess) st = VI_ERR_CUDA; else note_launch();
  }
  if (st == VI_OK) {
    TcArgs a{static_cast<const bf16*>(wpk), b, y, err};
    long long grid = sm_count();
    if (grid > pl.n_jobs) grid = pl.n_jobs;
    temporal_conv_tc_kernel<<<(unsigned)grid, TC_THREADS, pl.smem, stream>>>(tmx, pl, a);
    if (cudaGetLastError() != cudaSuccess) st = VI_ERR_CUDA; else note_launch();
  }
  if (cudaFreeAsync(wpk, stream) != cudaSuccess && st == VI_OK) st = VI_ERR_CUDA;
  return st;
}

}  // namespace vi
