// Temporal convolution with neighbour padding, all N clips on one GPU.
//
// Source: "Video-Infinity: Distributed Long Video Generation" (news.43zhubao.com
// write-up), conv-module paragraph.  Each clip is extended by the last n frames
// of the previous clip and the first n frames of the next (n = k/2, the conv's
// receptive field on one side), with zeros at the video ends, and convolved
// along frames with full C -> C channel mixing and a bias.  Since the
// neighbours' frames are exactly the adjacent frames of the [P][F][C] layout,
// the clip partition needs no data movement on one GPU: every output frame
// reads frames f-n .. f+n, and only the two video ends see zeros.
//
//   y[p,f,co] = b[co] + sum_t sum_ci w[co,ci,t] * x[p, f+t-n, ci]
//
// This file holds the CUDA-core path (fp32 I/O, and bf16 shapes the tensor-core
// path does not take): a CTA computes a 16-frame x 64-channel output tile of
// one position, staging x rows [f0-n, f0+16+n) and one tap of w per 32-channel
// slice in shared memory, fp32 accumulation.
#include "vi_internal.cuh"

namespace vi {

constexpr int CG_TF = 16;      // output frames per CTA
constexpr int CG_TCO = 64;     // output channels per CTA
constexpr int CG_TCI = 32;     // input channels per stage
constexpr int CG_MAXK = 15;    // largest kernel the staging buffer holds

template <typename T>
__global__ void __launch_bounds__(256) temporal_conv_generic(const T* __restrict__ x,
                                                             const T* __restrict__ w,
                                                             const T* __restrict__ b,
                                                             T* __restrict__ y, int F, int P,
                                                             int C, int k) {
  __shared__ float xs[CG_TF + CG_MAXK - 1][CG_TCI + 1];
  __shared__ float ws[CG_TCO][CG_TCI + 1];
  const int nft = (F + CG_TF - 1) / CG_TF, nct = (C + CG_TCO - 1) / CG_TCO;
  const int64_t id = blockIdx.x;
  const int ft = (int)(id % nft), ct = (int)((id / nft) % nct);
  const int64_t p = id / ((int64_t)nft * nct);
  const int f0 = ft * CG_TF, co0 = ct * CG_TCO, n = k / 2;
  const int tco = threadIdx.x % CG_TCO, tf = threadIdx.x / CG_TCO;   // 4 frame lanes
  const T* xp = x + p * F * C;
  float acc[CG_TF / 4];
#pragma unroll
  for (int j = 0; j < CG_TF / 4; ++j) acc[j] = 0.f;

  for (int ci0 = 0; ci0 < C; ci0 += CG_TCI) {
    __syncthreads();
    for (int e = threadIdx.x; e < (CG_TF + k - 1) * CG_TCI; e += blockDim.x) {
      const int r = e / CG_TCI, c = e % CG_TCI;
      const int f = f0 - n + r, ci = ci0 + c;
      xs[r][c] = (f >= 0 && f < F && ci < C) ? to_f32(xp[(int64_t)f * C + ci]) : 0.f;
    }
    for (int t = 0; t < k; ++t) {
      __syncthreads();
      for (int e = threadIdx.x; e < CG_TCO * CG_TCI; e += blockDim.x) {
        const int o = e / CG_TCI, c = e % CG_TCI;
        const int co = co0 + o, ci = ci0 + c;
        ws[o][c] = (co < C && ci < C) ? to_f32(w[((int64_t)co * C + ci) * k + t]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < CG_TCI; ++c) {
        const float wv = ws[tco][c];
#pragma unroll
        for (int j = 0; j < CG_TF / 4; ++j) acc[j] = fmaf(wv, xs[tf * (CG_TF / 4) + j + t][c], acc[j]);
      }
    }
  }
  const int co = co0 + tco;
  if (co < C) {
    const float bias = to_f32(b[co]);
#pragma unroll
    for (int j = 0; j < CG_TF / 4; ++j) {
      const int f = f0 + tf * (CG_TF / 4) + j;
      if (f < F) y[p * F * C + (int64_t)f * C + co] = from_f32<T>(acc[j] + bias);
    }
  }
}

template <typename T>
int temporal_conv_generic_launch(const T* x, const T* w, const T* b, T* y, int F, int P, int C,
                                 int k, cudaStream_t stream) {
  if (k > CG_MAXK) return VI_ERR_UNSUPPORTED;
  const int64_t blocks =
      (int64_t)P * ((F + CG_TF - 1) / CG_TF) * ((C + CG_TCO - 1) / CG_TCO);
  if (blocks > 0x7fffffff) return VI_ERR_UNSUPPORTED;
  temporal_conv_generic<T><<<(unsigned)blocks, 256, 0, stream>>>(x, w, b, y, F, P, C, k);
  VI_LAUNCHED();
  return VI_OK;
}

template int temporal_conv_generic_launch<float>(const float*, const float*, const float*, float*,
                                                 int, int, int, int, cudaStream_t);
template int temporal_conv_generic_launch<bf16>(const bf16*, const bf16*, const bf16*, bf16*, int,
                                                int, int, int, cudaStream_t);

}  // namespace vi
