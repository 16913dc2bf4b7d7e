// kernels_simt.cu - CUDA-core kernels of the DyRA forward.
//
//  * solve_kernel: per-instance ridge solve of Algorithm 1 line 12 ("DyRA:
//    Dynamic Residual Approximation for Efficient Matrix Multiplication in
//    DNNs", App. A; Sec. 2.4 uses a Cholesky solver for small k):
//      G_b = sum over row splits of L_b^T L_b  (+ lambda I, footnote 2 of Sec. 2.2)
//      T_b = sum over row splits of L_b^T X_b
//      T'_b = G_b^-1 T_b via Cholesky G_b = R R^T and two triangular solves.
//  * simt_gemm_kernel: strided, batched fp32 GEMM used by the fp32 plans
//    (fp32 accuracy needs plain FFMA; TF32 tensor cores would lose ~1e-3).
//  * pack_vp_kernel: builds [V | P]^T once at factor-load time.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"

namespace dyra {

namespace {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

constexpr int kSolveThreads = 128;

// grid (B, ceil(d_in / 128)); each CTA factors G_b itself (k <= 128, a few
// thousand flops) and solves for 128 columns of T_b, one column per thread.
template <typename TOut>
__global__ void __launch_bounds__(kSolveThreads)
    solve_kernel(const float* __restrict__ TG, int S, int B, int k, int d_in, float lambda,
                 TOut* __restrict__ Tp, int* status) {
  extern __shared__ float sm[];
  const int ldg = k + 1;
  float* G = sm;                     // k x (k+1): lower triangle becomes R
  float* Ycol = sm + k * ldg;        // k x 128: one column per thread
  __shared__ int bad;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int J = d_in + k;

  sm100::pdl_wait();

  if (tid == 0) bad = 0;
  for (int idx = tid; idx < k * k; idx += kSolveThreads) {
    const int i = idx / k, i2 = idx - (idx / k) * k;
    float g = 0.f;
    for (int s = 0; s < S; ++s)
      g += TG[(static_cast<size_t>(s) * B + b) * k * static_cast<size_t>(J) +
              static_cast<size_t>(i) * J + d_in + i2];
    G[i * ldg + i2] = g + (i == i2 ? lambda : 0.f);
  }
  __syncthreads();

  // Right-looking Cholesky, lower triangle: G = R R^T.
  for (int j = 0; j < k; ++j) {
    if (tid == 0) {
      const float d = G[j * ldg + j];
      if (!(d > 0.f) || !isfinite(d)) {
        bad = 1;
        G[j * ldg + j] = 1.f;
      } else {
        G[j * ldg + j] = sqrtf(d);
      }
    }
    __syncthreads();
    const float inv = 1.f / G[j * ldg + j];
    for (int i = j + 1 + tid; i < k; i += kSolveThreads) G[i * ldg + j] *= inv;
    __syncthreads();
    const int m = k - j - 1;  // trailing size
    for (int idx = tid; idx < m * m; idx += kSolveThreads) {
      const int i = j + 1 + idx / m, i2 = j + 1 + (idx - (idx / m) * m);
      if (i2 <= i) G[i * ldg + i2] -= G[i * ldg + j] * G[i2 * ldg + j];
    }
    __syncthreads();
  }

  const int col = blockIdx.y * kSolveThreads + tid;
  if (col < d_in) {
    for (int i = 0; i < k; ++i) {
      float t = 0.f;
      for (int s = 0; s < S; ++s)
        t += TG[(static_cast<size_t>(s) * B + b) * k * static_cast<size_t>(J) +
                static_cast<size_t>(i) * J + col];
      Ycol[i * kSolveThreads + tid] = t;
    }
    // R y = t
    for (int i = 0; i < k; ++i) {
      float acc = Ycol[i * kSolveThreads + tid];
      for (int q = 0; q < i; ++q) acc -= G[i * ldg + q] * Ycol[q * kSolveThreads + tid];
      Ycol[i * kSolveThreads + tid] = acc / G[i * ldg + i];
    }
    // R^T x = y
    for (int i = k - 1; i >= 0; --i) {
      float acc = Ycol[i * kSolveThreads + tid];
      for (int q = i + 1; q < k; ++q) acc -= G[q * ldg + i] * Ycol[q * kSolveThreads + tid];
      Ycol[i * kSolveThreads + tid] = acc / G[i * ldg + i];
    }
    const bool zero = bad != 0;
    for (int i = 0; i < k; ++i)
      Tp[(static_cast<size_t>(b) * k + i) * d_in + col] =
          from_f<TOut>(zero ? 0.f : Ycol[i * kSolveThreads + tid]);
  }
  if (tid == 0 && blockIdx.y == 0 && bad) atomicOr(status, sm100::kStatusPivot);
  __syncthreads();
  sm100::pdl_launch_dependents();
}

// C[b][m][n] (+)= sum_q A[b][m][q] * Bm[b][q][n] with arbitrary element strides.
constexpr int kGT = 64;   // tile
constexpr int kGK = 16;   // k step
template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256)
    simt_gemm_kernel(int M, int N, int K, const TA* __restrict__ A, int64_t am, int64_t ak,
                     int64_t ab, const TB* __restrict__ Bm, int64_t bk, int64_t bn, int64_t bb,
                     TC* __restrict__ C, int64_t cm, int64_t cn, int64_t cb, int accumulate) {
  __shared__ float As[kGK][kGT + 1];
  __shared__ float Bs[kGK][kGT + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * kGT, n0 = blockIdx.x * kGT;
  const int64_t batch = blockIdx.z;
  A += batch * ab;
  Bm += batch * bb;
  C += batch * cb;
  float acc[4][4] = {};
  for (int q0 = 0; q0 < K; q0 += kGK) {
    for (int idx = threadIdx.x; idx < kGK * kGT; idx += 256) {
      const int qq = idx / kGT, mm = idx % kGT;
      const int gm = m0 + mm, gq = q0 + qq;
      As[qq][mm] = (gm < M && gq < K) ? to_f<TA>(A[gm * am + gq * ak]) : 0.f;
      const int gn = n0 + mm;
      Bs[qq][mm] = (gn < N && gq < K) ? to_f<TB>(Bm[gq * bk + gn * bn]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int qq = 0; qq < kGK; ++qq) {
      float a[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[qq][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[qq][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      TC* dst = C + gm * cm + gn * cn;
      float v = acc[i][j];
      if (accumulate) v += to_f<TC>(*dst);
      *dst = from_f<TC>(v);
    }
  }
}

template <typename TA, typename TB, typename TC>
int gemm(int M, int N, int K, const TA* A, int64_t am, int64_t ak, int64_t ab, const TB* Bm,
         int64_t bk, int64_t bn, int64_t bb, TC* C, int64_t cm, int64_t cn, int64_t cb,
         int batches, int accumulate, cudaStream_t s) {
  if (M <= 0 || N <= 0 || batches <= 0) return 0;
  dim3 grid((N + kGT - 1) / kGT, (M + kGT - 1) / kGT, batches);
  simt_gemm_kernel<TA, TB, TC><<<grid, 256, 0, s>>>(M, N, K, A, am, ak, ab, Bm, bk, bn, bb, C,
                                                    cm, cn, cb, accumulate);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <typename T>
__global__ void pack_vp_kernel(const T* __restrict__ V, const T* __restrict__ P, T* __restrict__ VPt,
                               int d_in, int r, int k) {
  const int64_t total = static_cast<int64_t>(r + k) * d_in;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx / d_in);
    const int j = static_cast<int>(idx - static_cast<int64_t>(c) * d_in);
    VPt[idx] = c < r ? V[static_cast<int64_t>(j) * r + c] : P[static_cast<int64_t>(j) * k + (c - r)];
  }
}

}  // namespace

template <typename TOut>
int launch_solve(const float* TG, int splits, int64_t B, int k, int d_in, float lambda, TOut* Tp,
                 int* status, cudaStream_t s, bool pdl) {
  if (B == 0 || k == 0) return 0;
  const size_t smem = (static_cast<size_t>(k) * (k + 1) + static_cast<size_t>(k) * kSolveThreads) *
                      sizeof(float);
  auto kfn = solve_kernel<TOut>;
  static size_t configured = 48 * 1024;
  if (smem > configured) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -1;
    configured = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(B), static_cast<unsigned>((d_in + kSolveThreads - 1) / kSolveThreads));
  cfg.blockDim = dim3(kSolveThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kfn, TG, splits, static_cast<int>(B), k, d_in, lambda, Tp,
                            status) == cudaSuccess
             ? 0
             : -1;
}

template int launch_solve<float>(const float*, int, int64_t, int, int, float, float*, int*,
                                 cudaStream_t, bool);
template int launch_solve<__nv_bfloat16>(const float*, int, int64_t, int, int, float,
                                         __nv_bfloat16*, int*, cudaStream_t, bool);

template <typename T>
int launch_pack_vp(const T* V, const T* P, T* VPt, int d_in, int r, int k, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(r + k) * d_in;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 4096));
  pack_vp_kernel<T><<<blocks, 256, 0, s>>>(V, P, VPt, d_in, r, k);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template int launch_pack_vp<float>(const float*, const float*, float*, int, int, int, cudaStream_t);
template int launch_pack_vp<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                           __nv_bfloat16*, int, int, int, cudaStream_t);

// The fp32 forward: the same steps as the tensor-core path, each as a
// strided batched SIMT GEMM, with fp32 storage of every intermediate.
template <typename T>
int launch_simt_forward(const SimtForward<T>& a, const DeviceInfo&, cudaStream_t s) {
  const int64_t N = a.B * a.Trows;
  if (N == 0) return 0;
  const int rk = a.r + a.k;
  const int k = a.weight_only ? 0 : a.k;
  const int Bn = static_cast<int>(a.B);
  const int Tr = static_cast<int>(a.Trows);
  // [Z | L] = X [V | P]
  if (gemm(static_cast<int>(N), rk, a.d_in, a.X, a.d_in, 1, 0, a.VPt, 1, a.d_in, 0, a.ZL, rk, 1,
           0, 1, 0, s))
    return -1;
  if (k > 0) {
    const int J = a.d_in + k;
    // T_b = L_b^T X_b  -> TG[b][i][j], j < d_in
    if (gemm(k, a.d_in, Tr, a.ZL + a.r, 1, rk, static_cast<int64_t>(Tr) * rk, a.X, a.d_in, 1,
             static_cast<int64_t>(Tr) * a.d_in, a.TG, J, 1, static_cast<int64_t>(k) * J, Bn, 0, s))
      return -1;
    // G_b = L_b^T L_b -> TG[b][i][d_in + i']
    if (gemm(k, k, Tr, a.ZL + a.r, 1, rk, static_cast<int64_t>(Tr) * rk, a.ZL + a.r, rk, 1,
             static_cast<int64_t>(Tr) * rk, a.TG + a.d_in, J, 1, static_cast<int64_t>(k) * J, Bn, 0,
             s))
      return -1;
    if (launch_solve<T>(a.TG, 1, a.B, k, a.d_in, a.lambda, a.Tp, a.status, s, false)) return -1;
    // C = T' W_res^T  (B*k x d_out)
    if (gemm(Bn * k, a.d_out, a.d_in, a.Tp, a.d_in, 1, 0, a.W_res, 1, a.d_in, 0, a.Cm, a.d_out, 1,
             0, 1, 0, s))
      return -1;
  }
  // Y = Z U^T
  if (gemm(static_cast<int>(N), a.d_out, a.r, a.ZL, rk, 1, 0, a.U, 1, a.r, 0, a.Y, a.d_out, 1, 0,
           1, 0, s))
    return -1;
  if (k > 0) {
    // Y_b += L_b C_b
    if (gemm(Tr, a.d_out, k, a.ZL + a.r, rk, 1, static_cast<int64_t>(Tr) * rk, a.Cm, a.d_out, 1,
             static_cast<int64_t>(k) * a.d_out, a.Y, a.d_out, 1, static_cast<int64_t>(Tr) * a.d_out,
             Bn, 1, s))
      return -1;
  }
  return 0;
}

template int launch_simt_forward<float>(const SimtForward<float>&, const DeviceInfo&,
                                        cudaStream_t);
template int launch_simt_forward<__nv_bfloat16>(const SimtForward<__nv_bfloat16>&,
                                                const DeviceInfo&, cudaStream_t);

}  // namespace dyra
