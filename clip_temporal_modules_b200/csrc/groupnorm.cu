// GroupNorm with global statistics over all clips, for one GPU holding every
// clip of the video.
//
// Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
// write-up), GroupNorm-module paragraph.  There each device reduces its clip's
// group means into a global mean and then its spread about that mean into a
// global std.  With all clips on one GPU the per-clip step is simply a block
// of the grid: every block reduces a slice of rows, and the slices are merged
// into the global statistics by the last block to finish (no grid barrier).
//
// Pass 1 (gn_stats_*): one read of x.  Each thread accumulates, for the one or
//   two groups its 16-byte channel vector touches, the shifted sums
//   S1 = sum(x - K_g) and S2 = sum((x - K_g)^2) with K_g = x[0,0,first channel
//   of g] (the "shifted data" one-pass variance of Chan, Golub & LeVeque), in
//   fp32 over short runs folded into fp64.  Block totals go to scratch; the
//   last block (atomic ticket) merges them in fp64:
//     mu_g = K_g + S1/n,  var_g = S2/n - (S1/n)^2,
//   which is algebraically the pages' "global mean, then spread about it", and
//   turns them into per-channel coefficients m_c = mu_g (rounded to fp32),
//   a_c = gamma_c / sqrt(var_g+eps) and beta_c.
// Pass 2 (gn_apply_*): one read of x and one write of y = (x - m_c) a_c + beta_c
//   (subtracting first keeps a constant group exactly at beta).
// HBM traffic: 3 x |x|, the minimum for a two-pass normalisation of a tensor
// far larger than L2.
#include <math.h>

#include <mutex>

#include "ptx.cuh"
#include "vi_internal.cuh"

namespace vi {

constexpr int GN_MAX_GROUPS = 1024;
constexpr int GN_FOLD = 32;            // fp32 run length before folding into fp64

struct GnScratch {
  double* partials;        // [nparts][groups][3]: n, S1, S2
  float* coef;             // [C][4]: m_c, a_c, beta_c, 0
  unsigned int* ticket;    // blocks finished (reset to 0 by the last block)
  double* stats;           // [groups][2]: mu_g, var_g (kept for inspection)
};

// Where the apply pass takes its per-channel coefficients (m_c, a_c, beta_c):
// from coef, [C][4] floats written by the statistics pass, or (shard_stats
// != null) from W shards' per-group (mean, var) records, merged by each
// thread for its own channels exactly as gn_merge_coef does: mean = average
// of the means, var = average of (var_w + (mean_w - mean)^2).
template <typename T>
struct GnCoefSrc {
  const float* coef;
  const double* shard_stats;   // [W][groups][2]
  int W, groups, cg;
  const T* gamma;
  const T* beta;
  float eps;
};

template <typename T>
__device__ __forceinline__ void gn_coef_of(const GnCoefSrc<T>& src, int c, float& m, float& a,
                                           float& b) {
  if (!src.shard_stats) {
    m = src.coef[4 * c];
    a = src.coef[4 * c + 1];
    b = src.coef[4 * c + 2];
    return;
  }
  const int g = c / src.cg;
  double mean = 0.0;
  for (int w = 0; w < src.W; ++w) mean += src.shard_stats[((size_t)w * src.groups + g) * 2];
  mean /= src.W;
  double var = 0.0;
  for (int w = 0; w < src.W; ++w) {
    const double dm = src.shard_stats[((size_t)w * src.groups + g) * 2] - mean;
    var += src.shard_stats[((size_t)w * src.groups + g) * 2 + 1] + dm * dm;
  }
  var /= src.W;
  m = (float)mean;
  a = (float)((double)to_f32(src.gamma[c]) / sqrt(var + (double)src.eps));
  b = to_f32(src.beta[c]);
}

// Merge of all partial sums by the block that finishes last.  nparts partial
// records per group; red is the caller's shared buffer of GN_MAX_GROUPS rows.
template <typename T>
__device__ void gn_finalize(const GnScratch& s, int nparts, int groups, int C, int cg,
                            const T* __restrict__ x, const T* __restrict__ gamma,
                            const T* __restrict__ beta, float eps, double (*red)[3]) {
  for (int g = threadIdx.x; g < groups; g += blockDim.x) red[g][0] = red[g][1] = red[g][2] = 0.0;
  __syncthreads();
  // Every thread takes a strided share of (part, group) pairs.
  const int total = nparts * groups;
  double n = 0.0, s1 = 0.0, s2 = 0.0;
  int gcur = -1;
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int g = idx % groups;
    if (g != gcur) {
      if (gcur >= 0) {
        atomicAdd(&red[gcur][0], n); atomicAdd(&red[gcur][1], s1); atomicAdd(&red[gcur][2], s2);
      }
      gcur = g; n = s1 = s2 = 0.0;
    }
    const double* p = s.partials + (size_t)idx * 3;
    n += __ldcg(p); s1 += __ldcg(p + 1); s2 += __ldcg(p + 2);
  }
  if (gcur >= 0) {
    atomicAdd(&red[gcur][0], n); atomicAdd(&red[gcur][1], s1); atomicAdd(&red[gcur][2], s2);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const int g = c / cg;
    const double nn = red[g][0];
    const double m1 = red[g][1] / nn;
    const double var = fmax(red[g][2] / nn - m1 * m1, 0.0);
    const double mu = (double)to_f32(x[(size_t)g * cg]) + m1;
    // gamma/beta are null when only the statistics are wanted (a shard's pass).
    const double a = (gamma ? (double)to_f32(gamma[c]) : 1.0) / sqrt(var + (double)eps);
    s.coef[4 * c] = (float)mu;
    s.coef[4 * c + 1] = (float)a;
    s.coef[4 * c + 2] = beta ? to_f32(beta[c]) : 0.f;
    s.coef[4 * c + 3] = 0.f;
    if (c == g * cg) {
      s.stats[2 * g] = mu;
      s.stats[2 * g + 1] = var;
    }
  }
  if (threadIdx.x == 0) *s.ticket = 0u;
}

// Called by every block after writing its partial record(s): the block that
// takes the last ticket of nblocks merges the nparts records per group.
template <typename T>
__device__ __forceinline__ void gn_block_done(const GnScratch& s, int nblocks, int nparts,
                                              int groups, int C, int cg, const T* x,
                                              const T* gamma, const T* beta, float eps,
                                              double (*red)[3]) {
  __shared__ bool last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(s.ticket, 1u) == (unsigned)nblocks - 1u);
  __syncthreads();
  if (last) {
    __threadfence();
    gn_finalize<T>(s, nparts, groups, C, cg, x, gamma, beta, eps, red);
  }
}

// Vector path.  Persistent, one CTA per SM.  The tensor is cut into chunks of
// R_c whole rows (<= 32 KB); a producer warp streams chunks into a ring of
// GN_STAGES shared-memory stages with 1-D TMA bulk copies (up to 192 KB in
// flight per SM), and VPR x RB consumer threads read them back as 16-byte
// vectors.  Consumer thread (rr, j) always owns channel vector j (channels
// [jV, jV+V)) of rows rr, rr+RB, ... of a chunk, so it only ever touches the
// one or two groups that vector spans (checked on the host).
constexpr int GN_STAGES = 6;
constexpr int GN_CHUNK_MAX = 32768;

struct GnRing {
  int64_t rows;        // P * F
  int C;               // channels
  int rowbytes;        // C * sizeof(T)
  int rc;              // rows per chunk
  int64_t nchunks;
  int stage_bytes;     // rc * rowbytes (16B multiple)
  int VPR, RB;         // consumer layout
};

__device__ __forceinline__ uint32_t ring_stage(uint32_t base, const GnRing& g, int s) {
  return base + (uint32_t)s * g.stage_bytes;
}

template <typename T>
__global__ void __launch_bounds__(1024, 1) gn_stats_ring(const T* __restrict__ x, GnRing rg,
                                                         int cg, int groups, GnScratch s,
                                                         const T* __restrict__ gamma,
                                                         const T* __restrict__ beta, float eps,
                                                         unsigned int* err_word) {
  constexpr int V = VecOf<T>::n;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ double acc[GN_MAX_GROUPS][3];
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + GN_STAGES * rg.stage_bytes;     // full[S], empty[S]
  const int ncw = (blockDim.x >> 5) - 1;                        // consumer warps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int g = threadIdx.x; g < groups; g += blockDim.x) acc[g][0] = acc[g][1] = acc[g][2] = 0.0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < GN_STAGES; ++i) {
      mbar_init(bars + 8 * i, 1);
      mbar_init(bars + 8 * (GN_STAGES + i), ncw);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == ncw) {                                            // producer warp
    if (lane == 0) {
      int kl = 0;
      for (int64_t c = blockIdx.x; c < rg.nchunks; c += gridDim.x, ++kl) {
        const int st = kl % GN_STAGES, use = kl / GN_STAGES;
        if (use > 0 && !mbar_wait_bounded(bars + 8 * (GN_STAGES + st), (use - 1) & 1, err_word,
                                          VI_DEV_ERR_TMA_TIMEOUT))
          break;
        const int64_t r0 = c * rg.rc;
        const int nr = (int)min((int64_t)rg.rc, rg.rows - r0);
        const uint32_t bytes = (uint32_t)nr * rg.rowbytes;
        mbar_arrive_expect_tx(bars + 8 * st, bytes);
        bulk_load(ring_stage(base, rg, st), x + r0 * rg.C, bytes, bars + 8 * st);
      }
    }
  } else {
    const int t = threadIdx.x;
    const bool active = t < rg.VPR * rg.RB;
    const int j = t % rg.VPR, rr = t / rg.VPR;
    const int c0 = j * V;
    const int glo = c0 / cg;
    const int split = min(V, (glo + 1) * cg - c0);      // elements [0, split) are in glo
    const bool has_hi = split < V;
    // Per-element shift (the group's first value) and per-element running sums:
    // V independent dependency chains per thread, no per-element branching.
    float kk[V];
    {
      const float klo = active ? to_f32(x[(size_t)glo * cg]) : 0.f;
      const float khi = active && has_hi ? to_f32(x[(size_t)(glo + 1) * cg]) : 0.f;
#pragma unroll
      for (int e = 0; e < V; ++e) kk[e] = e < split ? klo : khi;
    }
    double d1lo = 0, d2lo = 0, d1hi = 0, d2hi = 0;
    int64_t nrows = 0;
    int kl = 0;
    for (int64_t c = blockIdx.x; c < rg.nchunks; c += gridDim.x, ++kl) {
      const int st = kl % GN_STAGES, use = kl / GN_STAGES;
      if (!mbar_wait_bounded(bars + 8 * st, use & 1, err_word, VI_DEV_ERR_TMA_TIMEOUT)) break;
      const int nr = (int)min((int64_t)rg.rc, rg.rows - c * rg.rc);
      if (active) {
        float s1[V], s2[V];
#pragma unroll
        for (int e = 0; e < V; ++e) s1[e] = s2[e] = 0.f;
        const uint32_t p0 = ring_stage(base, rg, st) + j * 16;
        int r = rr;
        for (; r + rg.RB < nr; r += 2 * rg.RB) {        // two rows per step
          float f[V], g[V];
          unpack(lds128(p0 + r * rg.rowbytes), f);
          unpack(lds128(p0 + (r + rg.RB) * rg.rowbytes), g);
#pragma unroll
          for (int e = 0; e < V; ++e) {
            const float a = f[e] - kk[e], b = g[e] - kk[e];
            s1[e] += a + b;
            s2[e] = fmaf(a, a, fmaf(b, b, s2[e]));
          }
          nrows += 2;
        }
        if (r < nr) {
          float f[V];
          unpack(lds128(p0 + r * rg.rowbytes), f);
#pragma unroll
          for (int e = 0; e < V; ++e) {
            const float a = f[e] - kk[e];
            s1[e] += a;
            s2[e] = fmaf(a, a, s2[e]);
          }
          ++nrows;
        }
        float a1lo = 0.f, a2lo = 0.f, a1hi = 0.f, a2hi = 0.f;
#pragma unroll
        for (int e = 0; e < V; ++e) {
          if (e < split) { a1lo += s1[e]; a2lo += s2[e]; }
          else { a1hi += s1[e]; a2hi += s2[e]; }
        }
        d1lo += a1lo; d2lo += a2lo; d1hi += a1hi; d2hi += a2hi;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (GN_STAGES + st));
    }
    if (active) {
      atomicAdd(&acc[glo][0], (double)(nrows * split));
      atomicAdd(&acc[glo][1], d1lo);
      atomicAdd(&acc[glo][2], d2lo);
      if (has_hi) {
        atomicAdd(&acc[glo + 1][0], (double)(nrows * (V - split)));
        atomicAdd(&acc[glo + 1][1], d1hi);
        atomicAdd(&acc[glo + 1][2], d2hi);
      }
    }
  }
  __syncthreads();
  for (int g = threadIdx.x; g < groups; g += blockDim.x) {
    double* p = s.partials + ((size_t)blockIdx.x * groups + g) * 3;
    p[0] = acc[g][0]; p[1] = acc[g][1]; p[2] = acc[g][2];
  }
  __syncthreads();
  gn_block_done<T>(s, gridDim.x, gridDim.x, groups, rg.C, cg, x, gamma, beta, eps, acc);
}

// y = (x - m_c) a_c + beta_c through the same ring: consumers rewrite each
// stage in place and the producer bulk-stores it back before reusing it.
// Chunks are visited last-first: the end of x, read last by the statistics
// pass, is the part most likely to still sit in L2.
template <typename T>
__global__ void __launch_bounds__(1024, 1) gn_apply_ring(const T* __restrict__ x,
                                                         T* __restrict__ y, GnRing rg,
                                                         const GnCoefSrc<T> csrc,
                                                         unsigned int* err_word) {
  constexpr int V = VecOf<T>::n;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + GN_STAGES * rg.stage_bytes;     // full[S], done[S]
  const int ncw = (blockDim.x >> 5) - 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < GN_STAGES; ++i) {
      mbar_init(bars + 8 * i, 1);
      mbar_init(bars + 8 * (GN_STAGES + i), ncw);
    }
    fence_barrier_init();
  }
  __syncthreads();
  auto chunk_of = [&](int kl) { return rg.nchunks - 1 - (blockIdx.x + (int64_t)kl * gridDim.x); };

  if (warp == ncw) {
    if (lane == 0) {
      const int nloc = (int)((rg.nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x);
      bool ok = true;
      auto store_back = [&](int kl) {        // stage of local chunk kl -> y
        const int st = kl % GN_STAGES;
        if (!mbar_wait_bounded(bars + 8 * (GN_STAGES + st), (kl / GN_STAGES) & 1, err_word,
                               VI_DEV_ERR_TMA_TIMEOUT))
          return false;
        const int64_t r0 = chunk_of(kl) * rg.rc;
        const int nr = (int)min((int64_t)rg.rc, rg.rows - r0);
        bulk_store(y + r0 * rg.C, ring_stage(base, rg, st), (uint32_t)nr * rg.rowbytes);
        bulk_commit();
        return true;
      };
      for (int kl = 0; kl < nloc && ok; ++kl) {
        const int st = kl % GN_STAGES;
        if (kl >= GN_STAGES) {
          ok = store_back(kl - GN_STAGES);
          bulk_wait_read_all();
          if (!ok) break;
        }
        const int64_t r0 = chunk_of(kl) * rg.rc;
        const int nr = (int)min((int64_t)rg.rc, rg.rows - r0);
        const uint32_t bytes = (uint32_t)nr * rg.rowbytes;
        mbar_arrive_expect_tx(bars + 8 * st, bytes);
        bulk_load(ring_stage(base, rg, st), x + r0 * rg.C, bytes, bars + 8 * st);
      }
      for (int kl = max(0, nloc - GN_STAGES); kl < nloc && ok; ++kl) ok = store_back(kl);
      bulk_wait_all();
    }
  } else {
    const int t = threadIdx.x;
    const bool active = t < rg.VPR * rg.RB;
    const int j = t % rg.VPR, rr = t / rg.VPR;
    const int c0 = j * V;
    float m[V], a[V], b[V];
#pragma unroll
    for (int e = 0; e < V; ++e) {
      m[e] = a[e] = b[e] = 0.f;
      if (active) gn_coef_of<T>(csrc, c0 + e, m[e], a[e], b[e]);
    }
    int kl = 0;
    for (int64_t c = blockIdx.x; c < rg.nchunks; c += gridDim.x, ++kl) {
      const int st = kl % GN_STAGES;
      if (!mbar_wait_bounded(bars + 8 * st, (kl / GN_STAGES) & 1, err_word,
                             VI_DEV_ERR_TMA_TIMEOUT))
        break;
      const int nr = (int)min((int64_t)rg.rc, rg.rows - chunk_of(kl) * rg.rc);
      if (active) {
        const uint32_t p0 = ring_stage(base, rg, st) + j * 16;
        for (int r = rr; r < nr; r += rg.RB) {
          float f[V];
          unpack(lds128(p0 + r * rg.rowbytes), f);
#pragma unroll
          for (int e = 0; e < V; ++e) f[e] = fmaf(f[e] - m[e], a[e], b[e]);
          sts128(p0 + r * rg.rowbytes, pack(f));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (GN_STAGES + st));
    }
  }
}

// Scalar path for channel groups narrower than a vector: block (g, part)
// reduces group g over its share of rows, one element per thread step.
template <typename T>
__global__ void __launch_bounds__(256) gn_stats_scalar(const T* __restrict__ x, int64_t rows,
                                                       int C, int cg, int groups, GnScratch s,
                                                       const T* __restrict__ gamma,
                                                       const T* __restrict__ beta, float eps) {
  const int g = blockIdx.x, part = blockIdx.y, nparts = gridDim.y;
  const int64_t r0 = rows * part / nparts, r1 = rows * (part + 1) / nparts;
  const int64_t nel = (r1 - r0) * cg;
  const float kg = to_f32(x[(size_t)g * cg]);
  double d1 = 0.0, d2 = 0.0;
  float a1 = 0.f, a2 = 0.f;
  int run = 0;
  for (int64_t e = threadIdx.x; e < nel; e += blockDim.x) {
    const int64_t r = r0 + e / cg;
    const int c = g * cg + (int)(e % cg);
    const float dv = to_f32(x[r * C + c]) - kg;
    a1 += dv; a2 = fmaf(dv, dv, a2);
    if (++run == GN_FOLD) { d1 += a1; d2 += a2; a1 = a2 = 0.f; run = 0; }
  }
  d1 += a1; d2 += a2;
  __shared__ double red[2][32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    d1 += __shfl_xor_sync(0xffffffffu, d1, o);
    d2 += __shfl_xor_sync(0xffffffffu, d2, o);
  }
  if ((threadIdx.x & 31) == 0) { red[0][threadIdx.x >> 5] = d1; red[1][threadIdx.x >> 5] = d2; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t1 = 0.0, t2 = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) { t1 += red[0][w]; t2 += red[1][w]; }
    // Part-major layout, as the vector path: partials[part][g].
    double* p = s.partials + ((size_t)part * groups + g) * 3;
    p[0] = (double)nel; p[1] = t1; p[2] = t2;
  }
  __shared__ double fin[GN_MAX_GROUPS][3];
  gn_block_done<T>(s, gridDim.x * gridDim.y, nparts, groups, C, cg, x, gamma, beta, eps, fin);
}

template <typename T>
__global__ void __launch_bounds__(256) gn_apply_scalar(const T* __restrict__ x, T* __restrict__ y,
                                                       int64_t n, int C,
                                                       const float* __restrict__ coef) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(e % C);
    y[e] = from_f32<T>(fmaf(to_f32(x[e]) - coef[4 * c], coef[4 * c + 1], coef[4 * c + 2]));
  }
}

// ---------------------------------------------------------------------------
// Host side.

struct GnPlan {
  bool ring;
  GnRing rg;
  int threads, blocks;         // ring path
  size_t smem;                 // ring path dynamic shared memory
  int parts;                   // scalar path: row slices per group
  int nparts;                  // partial records per group
};

template <typename T>
static GnPlan gn_plan(int64_t rows, int C, int groups) {
  constexpr int V = VecOf<T>::n;
  GnPlan pl{};
  const int cg = C / groups;
  const int VPR = C / V;
  const int rowbytes = C * (int)sizeof(T);
  bool ok = VPR <= 960 && rowbytes <= GN_CHUNK_MAX;
  for (int c0 = 0; ok && c0 < C; c0 += V)
    if ((c0 + V - 1) / cg - c0 / cg > 1) ok = false;
  pl.ring = ok;
  if (pl.ring) {
    GnRing& g = pl.rg;
    g.rows = rows;
    g.C = C;
    g.rowbytes = rowbytes;
    g.VPR = VPR;
    g.RB = 480 / VPR > 0 ? 480 / VPR : 1;
    g.rc = GN_CHUNK_MAX / rowbytes;
    g.stage_bytes = g.rc * rowbytes;
    g.nchunks = (rows + g.rc - 1) / g.rc;
    pl.threads = ((VPR * g.RB + 31) / 32) * 32 + 32;
    pl.smem = (size_t)GN_STAGES * g.stage_bytes + 16 * GN_STAGES;
    int64_t blocks = sm_count();
    if (blocks > g.nchunks) blocks = g.nchunks;
    pl.blocks = (int)blocks;
    pl.nparts = pl.blocks;
  } else {
    const int64_t per_group = (int64_t)(sm_count()) * 8 / groups + 1;
    const int64_t max_parts = (rows * cg + 255) / 256;
    pl.parts = (int)(per_group < max_parts ? per_group : max_parts);
    if (pl.parts < 1) pl.parts = 1;
    pl.nparts = pl.parts;
  }
  return pl;
}

// Carve the scratch block: ticket | stats | coef | partials (each 64B aligned).
static GnScratch gn_carve(void* base, int groups, int C) {
  GnScratch s;
  char* p = static_cast<char*>(base);
  s.ticket = reinterpret_cast<unsigned int*>(p);
  p += 64;
  s.stats = reinterpret_cast<double*>(p);
  p += ((sizeof(double) * 2 * groups + 63) / 64) * 64;
  s.coef = reinterpret_cast<float*>(p);
  p += ((sizeof(float) * 4 * (size_t)C + 63) / 64) * 64;
  s.partials = reinterpret_cast<double*>(p);
  return s;
}

template <typename T>
static size_t gn_scratch_bytes(int64_t rows, int C, int groups) {
  const GnPlan pl = gn_plan<T>(rows, C, groups);
  return 64 + ((sizeof(double) * 2 * groups + 63) / 64) * 64 +
         ((sizeof(float) * 4 * (size_t)C + 63) / 64) * 64 +
         sizeof(double) * 3 * (size_t)groups * pl.nparts;
}

// Enqueue both passes using caller-provided scratch (its ticket must read 0).
template <typename T>
static int gn_launch(const T* x, const T* gamma, const T* beta, T* y, int64_t rows, int C,
                     int groups, float eps, void* scratch, cudaStream_t stream) {
  const GnPlan pl = gn_plan<T>(rows, C, groups);
  const GnScratch s = gn_carve(scratch, groups, C);
  const int cg = C / groups;
  if (pl.ring) {
    unsigned int* err = device_error_word();
    if (!err) return VI_ERR_CUDA;
    VI_CUDA_TRY(cudaFuncSetAttribute(gn_stats_ring<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)pl.smem));
    VI_CUDA_TRY(cudaFuncSetAttribute(gn_apply_ring<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)pl.smem));
    gn_stats_ring<T><<<pl.blocks, pl.threads, pl.smem, stream>>>(x, pl.rg, cg, groups, s, gamma,
                                                                 beta, eps, err);
    VI_LAUNCHED();
    const GnCoefSrc<T> csrc{s.coef, nullptr, 0, groups, cg, nullptr, nullptr, 0.f};
    gn_apply_ring<T><<<pl.blocks, pl.threads, pl.smem, stream>>>(x, y, pl.rg, csrc, err);
    VI_LAUNCHED();
  } else {
    gn_stats_scalar<T><<<dim3(groups, pl.parts), 256, 0, stream>>>(x, rows, C, cg, groups, s,
                                                                  gamma, beta, eps);
    VI_LAUNCHED();
    const int64_t n = rows * C;
    int64_t blocks = (n + 255) / 256;
    if (blocks > (int64_t)sm_count() * 16) blocks = (int64_t)sm_count() * 16;
    gn_apply_scalar<T><<<(int)blocks, 256, 0, stream>>>(x, y, n, C, s.coef);
    VI_LAUNCHED();
  }
  return VI_OK;
}

// Statistics pass alone (for a consumer that applies the normalisation
// itself, such as the fused GroupNorm -> conv): fills the per-channel
// coefficients in `scratch` (whose ticket must read 0) and returns their
// address, [C][4] floats (m_c, a_c, beta_c, 0).
template <typename T>
int gn_stats_launch(const T* x, const T* gamma, const T* beta, int64_t rows, int C, int groups,
                    float eps, void* scratch, cudaStream_t stream, const float** coef,
                    double* stats_out) {
  const GnPlan pl = gn_plan<T>(rows, C, groups);
  GnScratch s = gn_carve(scratch, groups, C);
  if (stats_out) s.stats = stats_out;     // the last block writes (mean, var) there
  const int cg = C / groups;
  if (pl.ring) {
    unsigned int* err = device_error_word();
    if (!err) return VI_ERR_CUDA;
    VI_CUDA_TRY(cudaFuncSetAttribute(gn_stats_ring<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)pl.smem));
    gn_stats_ring<T><<<pl.blocks, pl.threads, pl.smem, stream>>>(x, pl.rg, cg, groups, s, gamma,
                                                                 beta, eps, err);
    VI_LAUNCHED();
  } else {
    gn_stats_scalar<T><<<dim3(groups, pl.parts), 256, 0, stream>>>(x, rows, C, cg, groups, s,
                                                                  gamma, beta, eps);
    VI_LAUNCHED();
  }
  *coef = s.coef;
  return VI_OK;
}

size_t gn_scratch_size_bf16(int64_t rows, int C, int groups) {
  return gn_scratch_bytes<bf16>(rows, C, groups);
}

template int gn_stats_launch<bf16>(const bf16*, const bf16*, const bf16*, int64_t, int, int, float,
                                   void*, cudaStream_t, const float**, double*);

// ---------------------------------------------------------------------------
// A video cut along frames over several GPUs (clip parallelism): each shard
// reduces its own rows (a6), the shards' statistics are exchanged and merged
// (a7), and each shard normalises its rows with the merged statistics (a8).

// a6 on one shard: per-group (mean, var) of the shard's rows, fp64, into
// stats [groups][2] (device memory), written by the statistics pass's last
// block itself.
template <typename T>
int gn_shard_stats(const T* x, int64_t rows, int C, int groups, double* stats,
                   cudaStream_t stream) {
  const size_t bytes = gn_scratch_bytes<T>(rows, C, groups);
  void* scratch = nullptr;
  VI_CUDA_TRY(scratch_alloc(&scratch, bytes, stream));
  const float* coef = nullptr;
  int st = cudaMemsetAsync(scratch, 0, 64, stream) == cudaSuccess ? VI_OK : VI_ERR_CUDA;
  if (st == VI_OK)
    st = gn_stats_launch<T>(x, nullptr, nullptr, rows, C, groups, 1e-5f, scratch, stream, &coef,
                            stats);
  if (scratch_free(scratch, stream) != cudaSuccess && st == VI_OK) st = VI_ERR_CUDA;
  return st;
}

// a7: merge W shards of equal row counts, shard_stats [W][groups][2] of
// (mean, var): mean = average of the means, var = average of (var_w +
// (mean_w - mean)^2) (the pooled biased variance); then the per-channel
// coefficients (m_c, a_c, beta_c, 0) of the normalisation.
template <typename T>
__global__ void gn_merge_coef(const double* __restrict__ shard_stats, int W, int groups, int C,
                              const T* __restrict__ gamma, const T* __restrict__ beta, float eps,
                              float* __restrict__ coef) {
  const int cg = C / groups;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < C; c += gridDim.x * blockDim.x) {
    const int g = c / cg;
    double mean = 0.0;
    for (int w = 0; w < W; ++w) mean += shard_stats[((size_t)w * groups + g) * 2];
    mean /= W;
    double var = 0.0;
    for (int w = 0; w < W; ++w) {
      const double dm = shard_stats[((size_t)w * groups + g) * 2] - mean;
      var += shard_stats[((size_t)w * groups + g) * 2 + 1] + dm * dm;
    }
    var /= W;
    const double a = (double)to_f32(gamma[c]) / sqrt(var + (double)eps);
    coef[4 * c] = (float)mean;
    coef[4 * c + 1] = (float)a;
    coef[4 * c + 2] = to_f32(beta[c]);
    coef[4 * c + 3] = 0.f;
  }
}

// a7 + a8 on one shard: merged statistics, then y = (x - m_c) a_c + beta_c.
// On the ring path every apply thread merges the shards' records for its own
// channels (one launch); the scalar path merges in a kernel of its own.
template <typename T>
int gn_shard_apply(const T* x, const double* shard_stats, int W, const T* gamma, const T* beta,
                   T* y, int64_t rows, int C, int groups, float eps, cudaStream_t stream) {
  const GnPlan pl = gn_plan<T>(rows, C, groups);
  if (pl.ring) {
    unsigned int* err = device_error_word();
    if (!err) return VI_ERR_CUDA;
    VI_CUDA_TRY(cudaFuncSetAttribute(gn_apply_ring<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)pl.smem));
    const GnCoefSrc<T> csrc{nullptr, shard_stats, W, groups, C / groups, gamma, beta, eps};
    gn_apply_ring<T><<<pl.blocks, pl.threads, pl.smem, stream>>>(x, y, pl.rg, csrc, err);
    VI_LAUNCHED();
    return VI_OK;
  }
  float* coef = nullptr;
  VI_CUDA_TRY(scratch_alloc(reinterpret_cast<void**>(&coef), sizeof(float) * 4 * (size_t)C,
                            stream));
  int st = VI_OK;
  gn_merge_coef<T><<<(C + 255) / 256, 256, 0, stream>>>(shard_stats, W, groups, C, gamma, beta,
                                                        eps, coef);
  if (cudaGetLastError() != cudaSuccess) st = VI_ERR_CUDA; else note_launch();
  if (st == VI_OK) {
    const int64_t n = rows * C;
    int64_t blocks = (n + 255) / 256;
    if (blocks > (int64_t)sm_count() * 16) blocks = (int64_t)sm_count() * 16;
    gn_apply_scalar<T><<<(int)blocks, 256, 0, stream>>>(x, y, n, C, coef);
    if (cudaGetLastError() != cudaSuccess) st = VI_ERR_CUDA; else note_launch();
  }
  if (scratch_free(coef, stream) != cudaSuccess && st == VI_OK) st = VI_ERR_CUDA;
  return st;
}

template int gn_shard_stats<bf16>(const bf16*, int64_t, int, int, double*, cudaStream_t);
template int gn_shard_apply<bf16>(const bf16*, const double*, int, const bf16*, const bf16*, bf16*,
                                  int64_t, int, int, float, cudaStream_t);

template <typename T>
int groupnorm_global(const T* x, const T* gamma, const T* beta, T* y, int64_t rows, int C,
                     int groups, float eps, cudaStream_t stream) {
  const size_t bytes = gn_scratch_bytes<T>(rows, C, groups);
  void* scratch = nullptr;
  VI_CUDA_TRY(scratch_alloc(&scratch, bytes, stream));
  cudaError_t e = cudaMemsetAsync(scratch, 0, 64, stream);
  int st = (e == cudaSuccess) ? gn_launch<T>(x, gamma, beta, y, rows, C, groups, eps, scratch,
                                             stream)
                              : VI_ERR_CUDA;
  if (scratch_free(scratch, stream) != cudaSuccess && st == VI_OK) st = VI_ERR_CUDA;
  return st;
}

template int groupnorm_global<float>(const float*, const float*, const float*, float*, int64_t,
                                     int, int, float, cudaStream_t);
template int groupnorm_global<bf16>(const bf16*, const bf16*, const bf16*, bf16*, int64_t, int,
                                    int, float, cudaStream_t);

}  // namespace vi

// ---------------------------------------------------------------------------
// Allocation-free entry point.
//
// Some callers cannot allocate device memory while they run: a plugin inside
// an inference engine that owns all device memory and forbids allocation in
// its execution step, or a service whose memory footprint is fixed when it
// starts.  vi_groupnorm_global takes its scratch from a stream-ordered pool, so
// those callers cannot use it.  vi_groupnorm_global_noalloc runs the same two
// kernels with its scratch in the file-scope array below instead; the caller
// still provides every input and output.
//
// The array is a module global: every GPU that loads libvi holds it until the
// process exits, and every call shares it (see include/vi.h).

namespace vi {

constexpr size_t GN_STATIC_SCRATCH_BYTES = size_t(1) << 20;      // 1 MiB
static __device__ __align__(256) unsigned char g_gn_static_scratch[GN_STATIC_SCRATCH_BYTES];

// Device address of g_gn_static_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device, with that device current, and cached.
static void* gn_static_scratch() {
  static std::mutex mu;
  static void* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gn_static_scratch) != cudaSuccess) return nullptr;
    cached[dev] = p;
  }
  return cached[dev];
}

}  // namespace vi

extern "C" int vi_groupnorm_global_noalloc(const void* x, const void* gamma, const void* beta,
                                           void* y, int F, int N, int P, int C, int groups,
                                           float eps, vi_stream_t stream) {
  using namespace vi;
  using T = bf16;
  // The argument checks of vi_groupnorm_global.
  if (F <= 0 || N <= 0 || P < 0 || C <= 0 || F % N != 0) return VI_ERR_INVALID_ARG;
  if ((double)P * (double)F * (double)C > 1.099511627776e12) return VI_ERR_UNSUPPORTED;
  if (groups <= 0 || C % groups != 0) return VI_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !isfinite(eps)) return VI_ERR_INVALID_ARG;
  if (groups > GN_MAX_GROUPS) return VI_ERR_UNSUPPORTED;
  if (P == 0) return VI_OK;                 // no positions: nothing to read or write
  if (!x || !gamma || !beta || !y) return VI_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(beta) || !aligned16(y))
    return VI_ERR_ALIGNMENT;
  if ((C * sizeof(T)) % 16 != 0) return VI_ERR_ALIGNMENT;
  const size_t bytes = (size_t)P * F * C * sizeof(T);
  if (y != x && overlaps(y, bytes, x, bytes)) return VI_ERR_INVALID_ARG;
  if (overlaps(y, bytes, gamma, C * sizeof(T)) || overlaps(y, bytes, beta, C * sizeof(T)))
    return VI_ERR_INVALID_ARG;
  // Scratch from the static array, never from an allocator.
  const int64_t rows = (int64_t)P * F;
  if (gn_scratch_bytes<T>(rows, C, groups) > GN_STATIC_SCRATCH_BYTES) return VI_ERR_UNSUPPORTED;
  void* scratch = gn_static_scratch();
  if (!scratch) return VI_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the completion ticket must
  // start at zero (the rest is fully rewritten before it is read).
  VI_CUDA_TRY(cudaMemsetAsync(scratch, 0, 64, s));
  return gn_launch<T>(static_cast<const T*>(x), static_cast<const T*>(gamma),
                      static_cast<const T*>(beta), static_cast<T*>(y), rows, C, groups, eps,
                      scratch, s);
}
