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
//   turns them into per-channel coefficients a_c = gamma_c / sqrt(var_g+eps),
//   b_c = beta_c - mu_g a_c.
// Pass 2 (gn_apply_*): one read of x and one write of y = x a_c + b_c.
// HBM traffic: 3 x |x|, the minimum for a two-pass normalisation of a tensor
// far larger than L2.
#include "vi_internal.cuh"

namespace vi {

constexpr int GN_THREADS_TARGET = 320;
constexpr int GN_MAX_GROUPS = 1024;
constexpr int GN_FOLD = 32;            // fp32 run length before folding into fp64

struct GnScratch {
  double* partials;        // [nparts][groups][3]: n, S1, S2
  float* coef;             // [C][2]: a_c, b_c
  unsigned int* ticket;    // blocks finished (reset to 0 by the last block)
  double* stats;           // [groups][2]: mu_g, var_g (kept for inspection)
};

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
    const double a = (double)to_f32(gamma[c]) / sqrt(var + (double)eps);
    s.coef[2 * c] = (float)a;
    s.coef[2 * c + 1] = (float)((double)to_f32(beta[c]) - mu * a);
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

// Vector path: blockDim = VPR * RB threads; thread (rr, j) owns channel vector
// j (channels [j*V, j*V+V)) of rows rr, rr+RB, ... of its block's share.  The
// vector spans at most two groups (checked on the host).
template <typename T>
__global__ void __launch_bounds__(1024) gn_stats_vec(const T* __restrict__ x, int64_t rows, int C,
                                                     int cg, int groups, int RB, GnScratch s,
                                                     const T* __restrict__ gamma,
                                                     const T* __restrict__ beta, float eps) {
  constexpr int V = VecOf<T>::n;
  __shared__ double acc[GN_MAX_GROUPS][3];
  const int VPR = C / V;
  for (int g = threadIdx.x; g < groups; g += blockDim.x) acc[g][0] = acc[g][1] = acc[g][2] = 0.0;
  __syncthreads();

  const int j = threadIdx.x % VPR, rr = threadIdx.x / VPR;
  if (rr < RB) {
    const int c0 = j * V;
    const int glo = c0 / cg;
    const int split = min(V, (glo + 1) * cg - c0);      // elements [0, split) are in glo
    const bool has_hi = split < V;
    const float klo = to_f32(x[(size_t)glo * cg]);
    const float khi = has_hi ? to_f32(x[(size_t)(glo + 1) * cg]) : 0.f;
    double d1lo = 0, d2lo = 0, d1hi = 0, d2hi = 0;
    int64_t nrows = 0;
    const int64_t step = (int64_t)gridDim.x * RB;
    int64_t r = (int64_t)blockIdx.x * RB + rr;
    while (r < rows) {
      float a1lo = 0.f, a2lo = 0.f, a1hi = 0.f, a2hi = 0.f;
      // A run of up to GN_FOLD rows, 4 loads in flight per thread.
      for (int it = 0; it < GN_FOLD && r < rows; it += 4) {
        uint4 u[4];
        int cnt = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (r + q * step < rows) {
            u[q] = *reinterpret_cast<const uint4*>(x + (r + q * step) * C + c0);
            ++cnt;
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q < cnt) {
            float f[V];
            unpack(u[q], f);
#pragma unroll
            for (int e = 0; e < V; ++e) {
              if (e < split) {
                const float dv = f[e] - klo;
                a1lo += dv; a2lo = fmaf(dv, dv, a2lo);
              } else {
                const float dv = f[e] - khi;
                a1hi += dv; a2hi = fmaf(dv, dv, a2hi);
              }
            }
          }
        }
        nrows += cnt;
        r += (int64_t)cnt * step;
      }
      d1lo += a1lo; d2lo += a2lo; d1hi += a1hi; d2hi += a2hi;
    }
    atomicAdd(&acc[glo][0], (double)(nrows * split));
    atomicAdd(&acc[glo][1], d1lo);
    atomicAdd(&acc[glo][2], d2lo);
    if (has_hi) {
      atomicAdd(&acc[glo + 1][0], (double)(nrows * (V - split)));
      atomicAdd(&acc[glo + 1][1], d1hi);
      atomicAdd(&acc[glo + 1][2], d2hi);
    }
  }
  __syncthreads();
  for (int g = threadIdx.x; g < groups; g += blockDim.x) {
    double* p = s.partials + ((size_t)blockIdx.x * groups + g) * 3;
    p[0] = acc[g][0]; p[1] = acc[g][1]; p[2] = acc[g][2];
  }
  __syncthreads();
  gn_block_done<T>(s, gridDim.x, gridDim.x, groups, C, cg, x, gamma, beta, eps, acc);
}

template <typename T>
__global__ void __launch_bounds__(1024) gn_apply_vec(const T* __restrict__ x, T* __restrict__ y,
                                                     int64_t rows, int C, int RB,
                                                     const float* __restrict__ coef) {
  constexpr int V = VecOf<T>::n;
  const int VPR = C / V;
  const int j = threadIdx.x % VPR, rr = threadIdx.x / VPR;
  if (rr >= RB) return;
  const int c0 = j * V;
  float a[V], b[V];
#pragma unroll
  for (int e = 0; e < V; ++e) {
    a[e] = coef[2 * (c0 + e)];
    b[e] = coef[2 * (c0 + e) + 1];
  }
  // Rows are visited last-first: the end of x, read last by the statistics
  // pass, is the part most likely to still sit in L2.
  const int64_t step = (int64_t)gridDim.x * RB;
  for (int64_t r = (int64_t)blockIdx.x * RB + rr; r < rows; r += 4 * step) {
    uint4 u[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (r + q * step < rows) u[q] = ld_stream(x + (rows - 1 - (r + q * step)) * C + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (r + q * step < rows) {
        float f[V];
        unpack(u[q], f);
#pragma unroll
        for (int e = 0; e < V; ++e) f[e] = fmaf(f[e], a[e], b[e]);
        st_stream(y + (rows - 1 - (r + q * step)) * C + c0, pack(f));
      }
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
    y[e] = from_f32<T>(fmaf(to_f32(x[e]), coef[2 * c], coef[2 * c + 1]));
  }
}

// ---------------------------------------------------------------------------
// Host side.

struct GnPlan {
  bool vec;
  int RB, threads, blocks;     // vector path
  int parts;                   // scalar path: row slices per group
  int nparts;                  // partial records per group
  size_t scratch_bytes;
};

template <typename T>
static GnPlan gn_plan(int64_t rows, int C, int groups) {
  constexpr int V = VecOf<T>::n;
  GnPlan pl{};
  const int cg = C / groups;
  const int VPR = C / V;
  bool span_ok = VPR <= 1024;
  for (int c0 = 0; span_ok && c0 < C; c0 += V)
    if ((c0 + V - 1) / cg - c0 / cg > 1) span_ok = false;
  pl.vec = span_ok;
  if (pl.vec) {
    pl.RB = GN_THREADS_TARGET / VPR > 0 ? GN_THREADS_TARGET / VPR : 1;
    pl.threads = VPR * pl.RB;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gn_stats_vec<T>, pl.threads, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t want = (rows + pl.RB - 1) / pl.RB;
    int64_t blocks = (int64_t)sm_count() * per_sm;
    if (blocks > want) blocks = want;
    pl.blocks = (int)(blocks > 0 ? blocks : 1);
    pl.nparts = pl.blocks;
  } else {
    const int64_t per_group = (int64_t)(sm_count()) * 8 / groups + 1;
    const int64_t max_parts = (rows * cg + 255) / 256;
    pl.parts = (int)(per_group < max_parts ? per_group : max_parts);
    if (pl.parts < 1) pl.parts = 1;
    pl.nparts = pl.parts;
  }
  pl.scratch_bytes = 256 + sizeof(double) * 3 * (size_t)groups * pl.nparts +
                     sizeof(float) * 2 * (size_t)C + sizeof(double) * 2 * (size_t)groups;
  return pl;
}

// Carve the scratch block: ticket | stats | coef | partials (each 16B aligned).
static GnScratch gn_carve(void* base, int groups, int C) {
  GnScratch s;
  char* p = static_cast<char*>(base);
  s.ticket = reinterpret_cast<unsigned int*>(p);
  p += 64;
  s.stats = reinterpret_cast<double*>(p);
  p += ((sizeof(double) * 2 * groups + 63) / 64) * 64;
  s.coef = reinterpret_cast<float*>(p);
  p += ((sizeof(float) * 2 * (size_t)C + 63) / 64) * 64;
  s.partials = reinterpret_cast<double*>(p);
  return s;
}

template <typename T>
static size_t gn_scratch_bytes(int64_t rows, int C, int groups) {
  const GnPlan pl = gn_plan<T>(rows, C, groups);
  return 64 + ((sizeof(double) * 2 * groups + 63) / 64) * 64 +
         ((sizeof(float) * 2 * (size_t)C + 63) / 64) * 64 +
         sizeof(double) * 3 * (size_t)groups * pl.nparts;
}

// Enqueue both passes using caller-provided scratch (ticket must read 0).
template <typename T>
static int gn_launch(const T* x, const T* gamma, const T* beta, T* y, int64_t rows, int C,
                     int groups, float eps, void* scratch, cudaStream_t stream) {
  const GnPlan pl = gn_plan<T>(rows, C, groups);
  const GnScratch s = gn_carve(scratch, groups, C);
  const int cg = C / groups;
  if (pl.vec) {
    gn_stats_vec<T><<<pl.blocks, pl.threads, 0, stream>>>(x, rows, C, cg, groups, pl.RB, s, gamma,
                                                         beta, eps);
    VI_CUDA_TRY(cudaGetLastError());
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gn_apply_vec<T>, pl.threads, 0);
    if (per_sm < 1) per_sm = 1;
    int64_t blocks = (int64_t)sm_count() * per_sm;
    const int64_t want = (rows + pl.RB - 1) / pl.RB;
    if (blocks > want) blocks = want;
    gn_apply_vec<T><<<(int)blocks, pl.threads, 0, stream>>>(x, y, rows, C, pl.RB, s.coef);
    VI_CUDA_TRY(cudaGetLastError());
  } else {
    gn_stats_scalar<T><<<dim3(groups, pl.parts), 256, 0, stream>>>(x, rows, C, cg, groups, s,
                                                                  gamma, beta, eps);
    VI_CUDA_TRY(cudaGetLastError());
    const int64_t n = rows * C;
    int64_t blocks = (n + 255) / 256;
    if (blocks > (int64_t)sm_count() * 16) blocks = (int64_t)sm_count() * 16;
    gn_apply_scalar<T><<<(int)blocks, 256, 0, stream>>>(x, y, n, C, s.coef);
    VI_CUDA_TRY(cudaGetLastError());
  }
  return VI_OK;
}

template <typename T>
int groupnorm_global(const T* x, const T* gamma, const T* beta, T* y, int64_t rows, int C,
                     int groups, float eps, cudaStream_t stream) {
  const size_t bytes = gn_scratch_bytes<T>(rows, C, groups);
  void* scratch = nullptr;
  VI_CUDA_TRY(cudaMallocAsync(&scratch, bytes, stream));
  cudaError_t e = cudaMemsetAsync(scratch, 0, 64, stream);
  int st = (e == cudaSuccess) ? gn_launch<T>(x, gamma, beta, y, rows, C, groups, eps, scratch,
                                             stream)
                              : VI_ERR_CUDA;
  if (cudaFreeAsync(scratch, stream) != cudaSuccess && st == VI_OK) st = VI_ERR_CUDA;
  return st;
}

template int groupnorm_global<float>(const float*, const float*, const float*, float*, int64_t,
                                     int, int, float, cudaStream_t);
template int groupnorm_global<bf16>(const bf16*, const bf16*, const bf16*, bf16*, int64_t, int,
                                    int, float, cudaStream_t);

}  // namespace vi
