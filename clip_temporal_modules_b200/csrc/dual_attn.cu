// Dual-domain temporal attention with all N clips of the video on one GPU.
//
// Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
// write-up), attention-module paragraph.  Every query frame of clip i attends,
// per spatial position and head, over one fixed key/value list: the clip's own
// L frames, the last n_pre frames of clip i-1 and the first n_post frames of
// clip i+1 (local context, absent at the video ends), and n_global frames
// sampled every floor(F/n_global) frames over the whole video (global
// context).  Duplicates are kept; the scale is 1/sqrt(d).
//
// On the pages each clip sits on its own GPU and the context frames arrive by
// an all_gather plus two neighbour exchanges.  Here the clip partition is the
// kernel grid: a CTA owns a run of clips of one (position, head), and the
// neighbours' frames are simply the adjacent rows of the [P][F][C] layout.
//
// Fast path (bf16, d = 64, n_global <= 16; clips of L = 16 frames with
// n_pre, n_post <= 16, or of L = 8 or 32 with n_pre, n_post <= 8):
//   CTA = (position p, block of 128 frames, head h), 8 warps.
//   One thread issues five TMA loads (128B-swizzled, one mbarrier), for a
//   window of H = 8 rows each side (H = 16 where a context exceeds 8):
//     Q   rows f0 .. f0+127                       16 KB
//     K,V rows f0-H .. f0+127+H ("window")        18 KB each (H = 8)
//     K,V rows j*stride, j < 16 ("global")         2 KB each
//   Rows outside [0, F) arrive as zeros and are masked out of the softmax.
//   Warp w owns query rows 16w .. 16w+15 (one clip of 16 frames, two of 8,
//   or half of one of 32) and the window rows of its clips' C_pre | own |
//   C_post (2H + 16 rows from 16w; 48 from 32(w/2) for clips of 32) plus the
//   16 global rows.  S = Q K^T and O = P V run on tensor cores
//   (mma.sync m16n8k16, bf16 in, fp32 accumulate: 24 + 24 instructions per
//   warp at H = 8), the softmax in fp32 registers with quad shuffles; P is
//   rounded to bf16 for the PV product and the row sums use the rounded
//   values.  O goes back through the Q buffer and one TMA store.
//   HBM traffic per token and head: q, k, v, out once each (4 x 128 B); the
//   halo and global rows are re-read by neighbouring CTAs from L2.
// Generic path (fp32 I/O, or shapes outside the fast path): one warp per
//   (position, head, query frame), keys walked in list order with an online
//   softmax in fp32 and expf; a clip's key list is staged in shared memory
//   once per CTA of (position, head, clip) where it fits (96 KB of K and V),
//   else read from global memory by every query.
#include <atomic>

#include "dual_attn_tile.cuh"
#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

// ---------------------------------------------------------------------------
// Generic path.

// Frame of entry t in clip i's key list (own, C_pre, C_post, C_global).
__device__ __forceinline__ int key_frame(int t, int i, int L, int N, int n_pre, int n_post,
                                         int gstride) {
  const int s = i * L;
  if (t < L) return s + t;
  t -= L;
  if (i > 0) {
    if (t < n_pre) return s - n_pre + t;
    t -= n_pre;
  }
  if (i < N - 1) {
    if (t < n_post) return s + L + t;
    t -= n_post;
  }
  return t * gstride;
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256) dual_attn_generic(const T* __restrict__ q,
                                                         const T* __restrict__ k,
                                                         const T* __restrict__ v,
                                                         T* __restrict__ out, int F, int N, int P,
                                                         int heads, int n_pre, int n_post,
                                                         int n_global, float scale) {
  constexpr int D = 32 * DPL;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= (int64_t)P * heads * F) return;
  const int f = (int)(wid % F);
  const int h = (int)((wid / F) % heads);
  const int64_t p = wid / ((int64_t)F * heads);
  const int C = heads * D, L = F / N, i = f / L;
  const int64_t pbase = p * F * C + (int64_t)h * D + lane * DPL;
  const int gstride = n_global > 0 ? F / n_global : 1;
  const int nk = L + (i > 0 ? n_pre : 0) + (i < N - 1 ? n_post : 0) + n_global;

  float qv[DPL], acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    qv[e] = to_f32(q[pbase + (int64_t)f * C + e]);
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int t = 0; t < nk; ++t) {
    const int64_t off = pbase + (int64_t)key_frame(t, i, L, N, n_pre, n_post, gstride) * C;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) dot = fmaf(qv[e], to_f32(k[off + e]), dot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float s = dot * scale;
    const float mn = fmaxf(m, s);
    const float alpha = expf(m - mn);      // exp(-inf) = 0 on the first key
    const float pe = expf(s - mn);
    l = l * alpha + pe;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pe, to_f32(v[off + e]), acc[e] * alpha);
    m = mn;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < DPL; ++e) out[pbase + (int64_t)f * C + e] = from_f32<T>(acc[e] * inv);
}

// The same computation with each clip's key list staged in shared memory:
// CTA = (position, head, clip), 4 warps.  The K and V rows of the clip's list
// (own, C_pre, C_post, C_global, in list order) are copied in once; then one
// warp per query frame of the clip walks them exactly as above (the same
// arithmetic in the same order: identical results), reading shared memory
// instead of re-reading the rows from L2 for every query.  nk_max: the
// longest key list of the video (rows of each staging buffer).
template <typename T, int DPL>
__global__ void __launch_bounds__(128) dual_attn_generic_staged(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ out,
    int F, int N, int heads, int n_pre, int n_post, int n_global, int nk_max, float scale) {
  constexpr int D = 32 * DPL;
  constexpr int VPR = D * (int)sizeof(T) / 16;   // 16-byte vectors per row
  extern __shared__ uint4 smem_vec[];
  T* sK = reinterpret_cast<T*>(smem_vec);
  T* sV = sK + (size_t)nk_max * D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = (int)(blockIdx.x % N);
  const int h = (int)((blockIdx.x / N) % heads);
  const int64_t p = blockIdx.x / ((int64_t)N * heads);
  const int C = heads * D, L = F / N;
  const int64_t base = p * F * C + (int64_t)h * D;
  const int gstride = n_global > 0 ? F / n_global : 1;
  const int nk = L + (i > 0 ? n_pre : 0) + (i < N - 1 ? n_post : 0) + n_global;
  for (int idx = threadIdx.x; idx < nk * VPR; idx += blockDim.x) {
    const int t = idx / VPR, c = idx % VPR;
    const int64_t off = base + (int64_t)key_frame(t, i, L, N, n_pre, n_post, gstride) * C;
    reinterpret_cast<uint4*>(sK + (size_t)t * D)[c] = reinterpret_cast<const uint4*>(k + off)[c];
    reinterpret_cast<uint4*>(sV + (size_t)t * D)[c] = reinterpret_cast<const uint4*>(v + off)[c];
  }
  __syncthreads();
  for (int fl = warp; fl < L; fl += 4) {
    const int64_t qo = base + (int64_t)(i * L + fl) * C + lane * DPL;
    float qv[DPL], acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      qv[e] = to_f32(q[qo + e]);
      acc[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < nk; ++t) {
      const T* kr = sK + (size_t)t * D + lane * DPL;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) dot = fmaf(qv[e], to_f32(kr[e]), dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float s = dot * scale;
      const float mn = fmaxf(m, s);
      const float alpha = expf(m - mn);      // exp(-inf) = 0 on the first key
      const float pe = expf(s - mn);
      l = l * alpha + pe;
      const T* vr = sV + (size_t)t * D + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pe, to_f32(vr[e]), acc[e] * alpha);
      m = mn;
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < DPL; ++e) out[qo + e] = from_f32<T>(acc[e] * inv);
  }
}

// Shared memory of the staged kernel: up to this much per CTA (K and V of the
// longest key list), else the unstaged kernel.
constexpr int GA_SMEM_MAX = 96 * 1024;

template <typename T>
static int ga_staged_prepare() {
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  VI_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    VI_CUDA_TRY(cudaFuncSetAttribute(dual_attn_generic_staged<T, 2>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, GA_SMEM_MAX));
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  return VI_OK;
}

template <typename T>
int dual_attn_generic_launch(const T* q, const T* k, const T* v, T* out, int F, int N, int P,
                             int heads, int d, int n_pre, int n_post, int n_global,
                             cudaStream_t stream) {
  if (d != 64) return VI_ERR_UNSUPPORTED;
  const float scale = 1.0f / sqrtf((float)d);
  const int L = F / N;
  const int nk_max = L + (N > 1 ? n_pre + n_post : 0) + n_global;
  const int64_t smem = 2 * (int64_t)nk_max * d * (int64_t)sizeof(T);
  const int64_t ctas = (int64_t)P * heads * N;
  if (smem <= GA_SMEM_MAX && ctas <= 0x7fffffff) {
    int st = ga_staged_prepare<T>();
    if (st != VI_OK) return st;
    dual_attn_generic_staged<T, 2><<<(unsigned)ctas, 128, (size_t)smem, stream>>>(
        q, k, v, out, F, N, heads, n_pre, n_post, n_global, nk_max, scale);
    VI_LAUNCHED();
    return VI_OK;
  }
  const int64_t warps = (int64_t)P * heads * F;
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffff) return VI_ERR_UNSUPPORTED;
  dual_attn_generic<T, 2><<<(unsigned)blocks, 256, 0, stream>>>(q, k, v, out, F, N, P, heads,
                                                                n_pre, n_post, n_global, scale);
  VI_LAUNCHED();
  return VI_OK;
}

// ---------------------------------------------------------------------------
// Fast path: TMA staging + mma.sync tensor-core tiles.

struct FaMaps {
  CUtensorMap q, k, v, kg, vg, o;
};

// N clips of the q map are computed; they are clips clip0 .. clip0 + N - 1 of
// a video of n_total clips (which decides the absent ends), and frame 0 of
// the q map is row kv_off of the k/v maps (0 for a whole video on one GPU,
// the halo width for a shard whose neighbours' frames are stacked around it).
// The grid covers the selected clip blocks of every (position, head): blocks
// [0, sel_lo) and [sel_hi0, sel_hi0 + n_sel - sel_lo).
//
// H: halo rows on each side of the CTA's 128 frames (the key list of a clip
// is H window rows before it, its own 16, H after it, then the 16 global
// frames: 2H + 32 keys, in n-tiles of 8).  LQ: frames per clip, 16 (one clip
// per warp) or 8 (two per warp, H = 8).
template <int H, int LQ = FA_L>
__global__ void __launch_bounds__(256) dual_attn_bf16_mma(const __grid_constant__ FaMaps maps,
                                                          int F, int N, int heads, int sel_lo,
                                                          int sel_hi0, int n_sel, int n_pre,
                                                          int n_post, int n_global,
                                                          float scale_log2, int kv_off, int clip0,
                                                          int n_total, unsigned int* err_word) {
  using Lay = FaLayout<H>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + Lay::OFF_Q, sKW = base + Lay::OFF_KW, sVW = base + Lay::OFF_VW;
  const uint32_t sKG = base + Lay::OFF_KG, sVG = base + Lay::OFF_VG, bar = base + Lay::OFF_BAR;

  const int sb = blockIdx.x % n_sel;
  const int blk = sb < sel_lo ? sb : sel_hi0 + (sb - sel_lo);
  const int h = (blockIdx.x / n_sel) % heads;
  const int p = blockIdx.x / (n_sel * heads);
  const int f0 = blk * FA_ROWS_Q;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t bytes = (FA_ROWS_Q + 2 * Lay::ROWS_W) * FA_ROW_BYTES +
                           (n_global > 0 ? 2 * FA_NG * FA_ROW_BYTES : 0);
    mbar_arrive_expect_tx(bar, bytes);
    tma_load_3d(sQ, &maps.q, h * 64, f0, p, bar);
    tma_load_3d(sKW, &maps.k, h * 64, f0 - H + kv_off, p, bar);
    tma_load_3d(sVW, &maps.v, h * 64, f0 - H + kv_off, p, bar);
    if (n_global > 0) {
      tma_load_3d(sKG, &maps.kg, h * 64, 0, p, bar);
      tma_load_3d(sVG, &maps.vg, h * 64, 0, p, bar);
    }
  }
  if (!mbar_wait_bounded(bar, 0, err_word, VI_DEV_ERR_TMA_TIMEOUT)) return;

  // The warp's (first) clip; clips of 8 frames come two to a warp.
  const int clip = (blk * FA_ROWS_Q + warp * 16) / LQ;
  if (clip < N) {
    const int gclip = clip0 + clip;              // index in the whole video
    fa_attend_warp<H, LQ>(sQ, sKW, sVW, sKG, sVG, warp, lane, gclip, n_total, n_pre, n_post,
                          n_global, scale_log2);
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_store_3d(&maps.o, sQ, h * 64, f0, p);
    tma_store_commit_and_drain();
  }
}

// Host: tensor maps over [P][F][C] bf16 with 128B swizzle.
bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                 CUtensorMapDataType dt);

// Raise the kernel's shared-memory limit once per device and kernel instance.
template <int H, int LQ>
static int fa_prepare() {
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  VI_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    // Idempotent, so concurrent first calls may both set it.
    VI_CUDA_TRY(cudaFuncSetAttribute(dual_attn_bf16_mma<H, LQ>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     FaLayout<H>::SMEM));
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  return VI_OK;
}

template <int H, int LQ>
static int fa_fast_launch(const bf16* q, const bf16* k, const bf16* v, bf16* out, int F, int N,
                          int P, int heads, int n_pre, int n_post, int n_global,
                          cudaStream_t stream) {
  const int C = heads * 64;
  FaMaps maps;
  const uint64_t dims[3] = {(uint64_t)C, (uint64_t)F, (uint64_t)P};
  const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)F * C * 2};
  const uint32_t boxQ[3] = {64, FA_ROWS_Q, 1}, boxW[3] = {64, FaLayout<H>::ROWS_W, 1};
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = encode_tmap(&maps.q, q, 3, dims, strides, boxQ, SW, BF) &&
            encode_tmap(&maps.k, k, 3, dims, strides, boxW, SW, BF) &&
            encode_tmap(&maps.v, v, 3, dims, strides, boxW, SW, BF) &&
            encode_tmap(&maps.o, out, 3, dims, strides, boxQ, SW, BF);
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
  int st = fa_prepare<H, LQ>();
  if (st != VI_OK) return st;
  const int cpb = FA_ROWS_Q / LQ;                 // clips per block of 128 frames
  const int nblk = (N + cpb - 1) / cpb;
  const int64_t grid = (int64_t)P * heads * nblk;
  if (grid > 0x7fffffff) return VI_ERR_UNSUPPORTED;
  const float scale_log2 = 1.4426950408889634f / 8.0f;    // log2(e) / sqrt(64)
  unsigned int* err = device_error_word();
  if (!err) return VI_ERR_CUDA;
  dual_attn_bf16_mma<H, LQ><<<(unsigned)grid, 256, FaLayout<H>::SMEM, stream>>>(
      maps, F, N, heads, nblk, 0, nblk, n_pre, n_post, n_global, scale_log2, 0, 0, N, err);
  VI_LAUNCHED();
  return VI_OK;
}

// The whole video on one GPU.  Clips of 16 frames: the narrower window (8
// rows each side) where both context sizes fit it, else the 16-row one; clips
// of 8 frames: the 8-row window, two clips per warp; of 32: the 8-row window,
// two warps per clip.
int dual_attn_bf16_fast(const bf16* q, const bf16* k, const bf16* v, bf16* out, int F, int N,
                        int P, int heads, int n_pre, int n_post, int n_global,
                        cudaStream_t stream) {
  if (F / N == 8)
    return fa_fast_launch<FA_HALO, 8>(q, k, v, out, F, N, P, heads, n_pre, n_post, n_global,
                                      stream);
  if (F / N == 32)
    return fa_fast_launch<FA_HALO, 32>(q, k, v, out, F, N, P, heads, n_pre, n_post, n_global,
                                       stream);
  if (n_pre <= FA_HALO && n_post <= FA_HALO)
    return fa_fast_launch<FA_HALO, FA_L>(q, k, v, out, F, N, P, heads, n_pre, n_post, n_global,
                                         stream);
  return fa_fast_launch<FA_HALO_MAX, FA_L>(q, k, v, out, F, N, P, heads, n_pre, n_post, n_global,
                                           stream);
}

// One shard of a video cut along frames (clip-parallel over several GPUs):
// q/out [P][F_loc][C] hold clips clip0 .. clip0 + N_loc - 1 of the video's N;
// k_ext/v_ext [P][F_loc + 2*FA_HALO][C] hold FA_HALO frames before the shard,
// the shard's frames and FA_HALO frames after it (rows past a video end are
// masked out, and must hold finite values); k_glob/v_glob [P][n_global][C]
// hold the video's global frames.
int dual_attn_bf16_shard(const bf16* q, const bf16* k_ext, const bf16* v_ext, const bf16* k_glob,
                         const bf16* v_glob, bf16* out, int F_loc, int N_loc, int clip0, int N,
                         int P, int heads, int n_pre, int n_post, int n_global, int part,
                         cudaStream_t stream) {
  const int C = heads * 64;
  const int F_ext = F_loc + 2 * FA_HALO;
  FaMaps maps;
  const uint64_t dims[3] = {(uint64_t)C, (uint64_t)F_loc, (uint64_t)P};
  const uint64_t strides[2] = {(uint64_t)C * 2, (uint64_t)F_loc * C * 2};
  const uint64_t edims[3] = {(uint64_t)C, (uint64_t)F_ext, (uint64_t)P};
  const uint64_t estrides[2] = {(uint64_t)C * 2, (uint64_t)F_ext * C * 2};
  const uint32_t boxQ[3] = {64, FA_ROWS_Q, 1}, boxW[3] = {64, FaLayout<FA_HALO>::ROWS_W, 1};
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = encode_tmap(&maps.q, q, 3, dims, strides, boxQ, SW, BF) &&
            encode_tmap(&maps.k, k_ext, 3, edims, estrides, boxW, SW, BF) &&
            encode_tmap(&maps.v, v_ext, 3, edims, estrides, boxW, SW, BF) &&
            encode_tmap(&maps.o, out, 3, dims, strides, boxQ, SW, BF);
  if (n_global > 0) {
    const uint64_t gdims[3] = {(uint64_t)C, (uint64_t)n_global, (uint64_t)P};
    const uint64_t gstrides[2] = {(uint64_t)C * 2, (uint64_t)n_global * C * 2};
    const uint32_t boxG[3] = {64, FA_NG, 1};
    ok = ok && encode_tmap(&maps.kg, k_glob, 3, gdims, gstrides, boxG, SW, BF) &&
         encode_tmap(&maps.vg, v_glob, 3, gdims, gstrides, boxG, SW, BF);
  } else {
    maps.kg = maps.k;
    maps.vg = maps.v;
  }
  if (!ok) return VI_ERR_CUDA;
  int st = fa_prepare<FA_HALO, FA_L>();
  if (st != VI_OK) return st;
  const int nblk = (N_loc + FA_CLIPS - 1) / FA_CLIPS;
  // Interior blocks [a, b): their k/v window (8 rows on each side of the
  // block) lies inside the shard's own frames.  The others are the boundary.
  const int a = nblk < 1 ? nblk : 1, b = nblk - 1 > a ? nblk - 1 : a;
  int sel_lo = nblk, sel_hi0 = 0, n_sel = nblk;
  if (part == VI_PART_INTERIOR) {
    sel_lo = 0; sel_hi0 = a; n_sel = b - a;
  } else if (part == VI_PART_BOUNDARY) {
    sel_lo = a; sel_hi0 = b; n_sel = a + (nblk - b);
  }
  if (n_sel == 0) return VI_OK;              // nothing in this part
  const int64_t grid = (int64_t)P * heads * n_sel;
  if (grid > 0x7fffffff) return VI_ERR_UNSUPPORTED;
  const float scale_log2 = 1.4426950408889634f / 8.0f;    // log2(e) / sqrt(64)
  unsigned int* err = device_error_word();
  if (!err) return VI_ERR_CUDA;
  dual_attn_bf16_mma<FA_HALO, FA_L><<<(unsigned)grid, 256, FaLayout<FA_HALO>::SMEM, stream>>>(
      maps, F_loc, N_loc, heads, sel_lo, sel_hi0, n_sel, n_pre, n_post, n_global, scale_log2,
      FA_HALO, clip0, N, err);
  VI_LAUNCHED();
  return VI_OK;
}

// Clips of 16 frames with up to 16 context frames on each side, or of 8 or
// 32 with up to 8; at most 16 global frames; d = 64.
bool dual_attn_fast_ok(int F, int N, int d, int n_pre, int n_post, int n_global) {
  const int L = F / N;
  const int ctx = L == FA_L ? FA_HALO_MAX : (L == 8 || L == 32) ? FA_HALO : -1;
  return d == 64 && ctx >= 0 && n_pre <= ctx && n_post <= ctx && n_global <= FA_NG;
}

// A shard's k/v storage carries FA_HALO rows of its neighbours on each side.
bool dual_attn_shard_ok(int L, int d, int n_pre, int n_post, int n_global) {
  return d == 64 && L == FA_L && n_pre <= FA_HALO && n_post <= FA_HALO && n_global <= FA_NG;
}

template int dual_attn_generic_launch<float>(const float*, const float*, const float*, float*,
                                             int, int, int, int, int, int, int, int,
                                             cudaStream_t);
template int dual_attn_generic_launch<bf16>(const bf16*, const bf16*, const bf16*, bf16*, int,
                                            int, int, int, int, int, int, int, cudaStream_t);

}  // namespace vi
