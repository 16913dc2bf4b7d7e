// kernels_simt.cu - CUDA-core kernels of the DyRA forward.
//
//  * solve_kernel / solve_ldl_kernel (fp32 plans): per-instance ridge solve of
//    the right factor in Algorithm 1, procedure Inference ("DyRA: Dynamic
//    Residual Approximation for Efficient Matrix Multiplication in DNNs",
//    App. A; Sec. 2.4 uses a Cholesky solver for small k):
//      G_b = sum over row splits of L_b^T L_b  (+ lambda I, footnote 2 of Sec. 2.2)
//      T_b = sum over row splits of L_b^T X_b
//      T'_b = G_b^-1 T_b (Cholesky with two triangular solves, or the blocked
//      LDL^T of ldl_panel.cuh for k <= 64).
//  * ltilde_kernel / ltilde_general_kernel (bf16 plans): L~_b = L_b G_b^-1
//    over L, the same solve applied on the side of L.
//  * simt_gemm_kernel: strided, batched fp32 GEMM used by the fp32 plans
//    (fp32 accuracy needs plain FFMA; TF32 tensor cores would lose ~1e-3).
//  * pack_vp_kernel: builds [V | P]^T once at factor-load time.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstddef>

#include "internal.h"
#include "ldl_panel.cuh"
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

// General variant (any k <= 128). grid (B, ceil(d_in / 128)); each CTA
// factors G_b itself (Cholesky in shared memory) and solves for 128 columns
// of T_b, one column per thread.
template <typename TOut>
__global__ void __launch_bounds__(kSolveThreads)
    solve_kernel(const float* __restrict__ TG, int S, int B, int k, int d_in, float lambda,
                 TOut* __restrict__ Tp, int* status, float alpha) {
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
      if (sm100::in_bounds(status, (static_cast<size_t>(b) * k + i) * d_in + col, 1,
                           static_cast<size_t>(B) * k * d_in))
        Tp[(static_cast<size_t>(b) * k + i) * d_in + col] =
            from_f<TOut>(zero ? 0.f : alpha * Ycol[i * kSolveThreads + tid]);
  }
  if (tid == 0 && blockIdx.y == 0 && bad) atomicOr(status, sm100::kStatusPivot);
  __syncthreads();
  sm100::pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// Fast path for k <= 64. grid (B, ceil(d_in / 128)), 256 threads; each CTA
// handles a 128-column chunk of T_b. G_b + lambda I = Lt D Lt^T by the panel
// elimination of ldl_panel.cuh gives M = Lt^-1 and D; the CTA then applies
// T' = M^T D^-1 (M T) to its chunk: two small products, no sequential
// dependency (same accuracy as the two triangular solves). Every CTA factors
// G_b itself (the CUDA-core path of fp32 plans). The T chunk's first split
// is loaded before the factorisation and waits in registers while it runs;
// the other splits are added afterwards.
constexpr int kSolveThreads2 = 256;
constexpr int kSolveCols = 128;  // columns of T_b per CTA
enum SolveMode { kSolveSelf = 0, kSolveShared = 1, kSolveGiven = 2 };

template <int KMAX>
struct SolveSmem {
  static constexpr int LDM = KMAX + 4;  // M rows, 16-byte aligned
  float Tc[KMAX * kSolveCols];          // T chunk
  float Us[KMAX * kSolveCols];          // D^-1 M T
  float Mr[KMAX * LDM];                 // Mr[i][q] = M[i][q]
  float Mc[KMAX * LDM];                 // Mc[q][i] = M[i][q]
  float dinv[KMAX];
  LdlBlockScratch<KMAX> ldl;
  int bad;
};

template <typename TOut, int KMAX>
__global__ void __launch_bounds__(kSolveThreads2)
    solve_ldl_kernel(const float* __restrict__ TG, int S, int B, int k, int d_in, float lambda,
                     TOut* __restrict__ Tp, int* status,
                     unsigned long long* trace, float alpha) {
  using Sm = SolveSmem<KMAX>;
  constexpr int LDG = LdlBlockScratch<KMAX>::LD;
  extern __shared__ __align__(16) unsigned char smem_bytes[];
  Sm& sm = *reinterpret_cast<Sm*>(smem_bytes);
  constexpr int GPT = KMAX * KMAX / kSolveThreads2;
  constexpr int TPT = KMAX * kSolveCols / kSolveThreads2;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int rg = tid >> 5, cg = tid & 31;
  const int J = d_in + k;
  const int c0 = blockIdx.y * kSolveCols;
  const size_t inst = static_cast<size_t>(k) * J;
  unsigned long long* const tr =
      trace ? trace + (blockIdx.y * gridDim.x + blockIdx.x) % kTraceCtas * kTraceSlots : nullptr;
  if (tr && tid == 0) tr[0] = sm100::globaltimer_ns();
  sm100::pdl_wait();
  if (tr && tid == 0) tr[2] = sm100::globaltimer_ns();
  // The next stage may be launched now: its blocks wait for this grid's
  // results in their own pdl_wait and take SMs as these blocks leave.
  sm100::pdl_launch_dependents();

  // ---- 1. loads: the first split of the T chunk (kept in registers until
  // after the factorisation), then G_b
  const float* part = TG + static_cast<size_t>(b) * inst;
  float t[TPT];
#pragma unroll
  for (int u = 0; u < TPT; ++u) {
    const int idx = tid + u * kSolveThreads2;
    const int i = idx / kSolveCols, c = idx % kSolveCols;
    t[u] = (i < k && c0 + c < d_in) ? part[static_cast<size_t>(i) * J + c0 + c] : 0.f;
  }
  {
    float g[GPT];
#pragma unroll
    for (int u = 0; u < GPT; ++u) {
      const int idx = tid + u * kSolveThreads2;
      const int i = idx / KMAX, q = idx % KMAX;
      g[u] = (i < k && q < k) ? part[static_cast<size_t>(i) * J + d_in + q] : 0.f;
    }
    for (int sp = 1; sp < S; ++sp) {
      const float* ps = TG + (static_cast<size_t>(sp) * B + b) * inst;
#pragma unroll
      for (int u = 0; u < GPT; ++u) {
        const int idx = tid + u * kSolveThreads2;
        const int i = idx / KMAX, q = idx % KMAX;
        if (i < k && q < k) g[u] += ps[static_cast<size_t>(i) * J + d_in + q];
      }
    }
#pragma unroll
    for (int u = 0; u < GPT; ++u) {
      const int idx = tid + u * kSolveThreads2;
      const int i = idx / KMAX, q = idx % KMAX;
      sm.ldl.Gs[i * LDG + q] =
          (i < k && q < k) ? g[u] + (i == q ? lambda : 0.f) : (i == q ? 1.f : 0.f);
    }
    if (tid == 0) sm.bad = 0;
  }
  __syncthreads();
  if (tr && tid == 0) tr[3] = sm100::globaltimer_ns();

  // ---- 2. the factorisation
  {
    const bool ok = ldl_blocked<KMAX, kSolveThreads2>(
        sm.ldl, k, tid, [] { __syncthreads(); },
        [&](int i, int q, float v) {
          sm.Mr[i * Sm::LDM + q] = v;
          sm.Mc[q * Sm::LDM + i] = v;
        },
        [&](int j, float v) { sm.dinv[j] = v; }, tr ? tr + 40 : nullptr);
    if (tid == 0 && !ok) sm.bad = 1;
  }
  // the remaining splits of the T chunk
  for (int sp = 1; sp < S; ++sp) {
    const float* ps = TG + (static_cast<size_t>(sp) * B + b) * inst;
#pragma unroll
    for (int u = 0; u < TPT; ++u) {
      const int idx = tid + u * kSolveThreads2;
      const int i = idx / kSolveCols, c = idx % kSolveCols;
      if (i < k && c0 + c < d_in) t[u] += ps[static_cast<size_t>(i) * J + c0 + c];
    }
  }
#pragma unroll
  for (int u = 0; u < TPT; ++u) sm.Tc[tid + u * kSolveThreads2] = t[u];
  __syncthreads();
  if (tr && tid == 0) tr[4] = sm100::globaltimer_ns();

  // ---- 3. T' = M^T D^-1 (M T): RPT rows x 4 columns per thread
  constexpr int RPT = KMAX / 8;
  float acc[RPT][4];
#pragma unroll
  for (int u = 0; u < RPT; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
  // M is unit lower triangular: rows rg*RPT.. need q <= their index only.
  const int qmax = min(k, (rg + 1) * RPT);
#pragma unroll 4
  for (int q = 0; q < qmax; ++q) {  // U = M T, M[i][q] = Mc[q][i]
    const float4 t4 = *reinterpret_cast<const float4*>(&sm.Tc[q * kSolveCols + 4 * cg]);
#pragma unroll
    for (int u = 0; u < RPT; u += 4) {
      const float4 m4 = *reinterpret_cast<const float4*>(&sm.Mc[q * Sm::LDM + rg * RPT + u]);
      const float m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        acc[u + w][0] = fmaf(m[w], t4.x, acc[u + w][0]);
        acc[u + w][1] = fmaf(m[w], t4.y, acc[u + w][1]);
        acc[u + w][2] = fmaf(m[w], t4.z, acc[u + w][2]);
        acc[u + w][3] = fmaf(m[w], t4.w, acc[u + w][3]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const int i = rg * RPT + u;
    const float di = sm.dinv[i];
    *reinterpret_cast<float4*>(&sm.Us[i * kSolveCols + 4 * cg]) =
        make_float4(acc[u][0] * di, acc[u][1] * di, acc[u][2] * di, acc[u][3] * di);
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
  }
  __syncthreads();
#pragma unroll 4
  for (int q = rg * RPT; q < k; ++q) {  // T' = M^T V, M[q][i] = Mr[q][i], q >= i
    const float4 v4 = *reinterpret_cast<const float4*>(&sm.Us[q * kSolveCols + 4 * cg]);
#pragma unroll
    for (int u = 0; u < RPT; u += 4) {
      const float4 m4 = *reinterpret_cast<const float4*>(&sm.Mr[q * Sm::LDM + rg * RPT + u]);
      const float m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        acc[u + w][0] = fmaf(m[w], v4.x, acc[u + w][0]);
        acc[u + w][1] = fmaf(m[w], v4.y, acc[u + w][1]);
        acc[u + w][2] = fmaf(m[w], v4.z, acc[u + w][2]);
        acc[u + w][3] = fmaf(m[w], v4.w, acc[u + w][3]);
      }
    }
  }
  if (tr && tid == 0) tr[5] = sm100::globaltimer_ns();
  const bool zero = sm.bad != 0;
  const int col = c0 + 4 * cg;
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const int i = rg * RPT + u;
    if (i >= k) continue;
    TOut* dst = Tp + (static_cast<size_t>(b) * k + i) * d_in + col;
#pragma unroll
    for (int v = 0; v < 4; ++v)
      if (col + v < d_in &&
          sm100::in_bounds(status, (dst - Tp) + v, 1, static_cast<size_t>(B) * k * d_in))
        dst[v] = from_f<TOut>(zero ? 0.f : alpha * acc[u][v]);
  }
  if (tid == 0 && blockIdx.y == 0 && zero) atomicOr(status, sm100::kStatusPivot);
  __syncthreads();
  if (tr && tid == 0) tr[8] = sm100::globaltimer_ns();
}

// ---------------------------------------------------------------------------
// Ridge solve on the side of L (bf16 plans): L~_b = L_b G_b^-1, written over
// L_b. With it the correction of Algorithm 1 ("DyRA", App. A, procedure
// Inference) is regrouped as
//   L_b C_b = L_b G_b^-1 (T_b W_res^T) = L~_b Q_b,   Q_b = T_b W_res^T,
// the same product up to rounding: the GEMM for Q_b needs T_b only, so it runs
// while this kernel factors G_b, and the output stage multiplies L~ by Q.
// grid (B, ceil(T / rows)), 256 threads, 256 (KMAX = 32) or 128 (KMAX = 64)
// rows of L_b per block: G_b + lambda I = Lt D Lt^T by the blocked elimination
// of ldl_panel.cuh gives M = Lt^-1 and D, then G_b^-1 = M^T D^-1 M is formed
// once (fp32) and the block's rows are multiplied by it in a register-tiled
// product (G_b is symmetric, so a row times G_b^-1 is G_b^-1 times the row).
// Who factors: every CTA (kSolveSelf), or the instance's first CTA, which
// publishes G_b^-1 and a failure flag for the others (kSolveShared), or no
// CTA: another kernel (the Newton-Schulz iteration) published the records
// (kSolveGiven).
// defer_wait: the grid launched just before this one (the GEMM for Q) has
// already waited for the Gram stage before letting this grid start, so this
// grid reads G and L at once and waits for that grid only before it exits
// (the output stage then relies on both). The next grid may start at once.
constexpr int kLtThreads = 256;

// Rows of L_b per block: 256 for KMAX = 32, 128 for KMAX = 64 (the staged
// rows then fit the factorisation's scratch, which is free by then).
template <int KMAX>
__host__ __device__ constexpr int lt_rows() {
  return KMAX <= 32 ? 256 : 128;
}

template <int KMAX>
struct LtSmem {
  static constexpr int kVS = KMAX + 8;  // staged row stride (bf16): 16-byte rows, spread banks
  LdlBlockScratch<KMAX> ldl;            // after the factorisation: Gs = M, Wb = G^-1 (stride KMAX)
  // the block's rows of L_b (bf16, stride kVS); for KMAX = 64 they are staged
  // over ldl.Gs and ldl.Mb instead, once G^-1 is formed
  alignas(16) __nv_bfloat16 Vs[KMAX <= 32 ? lt_rows<KMAX>() * kVS : 8];
};
static_assert(2 * sizeof(float) * 64 * 65 >= sizeof(__nv_bfloat16) * 128 * 72,
              "KMAX = 64: the staged rows fit over Gs and Mb");
// 16-byte copies into the staged rows and float4 accesses to M and G^-1
static_assert(offsetof(LtSmem<32>, Vs) % 16 == 0 && offsetof(LtSmem<64>, Vs) % 16 == 0,
              "staged rows 16-byte aligned");
static_assert(offsetof(LdlBlockScratch<32>, Wb) % 16 == 0 &&
                  offsetof(LdlBlockScratch<64>, Wb) % 16 == 0 &&
                  offsetof(LdlBlockScratch<64>, Mb) % 16 == 0,
              "G^-1 and the KMAX = 64 staging 16-byte aligned");

// 152 registers: a block fits on an SM beside a block of the rank-k factor
// GEMM. Registers come from the SM's four sub-partitions, 16K each, and a
// sub-partition may hold two warps of each block: 2 x 152 x 32 + 2 x 104 x 32
// = 16384 (the GEMM's warps take up to 104 registers).
template <int KMAX, int MODE>
__global__ void __maxnreg__(152)
    ltilde_kernel(const float* __restrict__ G, __nv_bfloat16* L, __nv_bfloat16* Llo, float* MD,
                  int* flags, int T, int k, float lambda, float alpha, int* status, int defer_wait,
                  unsigned long long* trace) {
  using Sm = LtSmem<KMAX>;
  constexpr int LD = LdlBlockScratch<KMAX>::LD;
  constexpr int ROWS = lt_rows<KMAX>();
  constexpr int VS = Sm::kVS;
  constexpr int NB = KMAX / 16;
  extern __shared__ __align__(16) unsigned char smem_bytes[];
  Sm& sm = *reinterpret_cast<Sm*>(smem_bytes);
  float* const Ma = sm.ldl.Gs;  // M, row-major, stride KMAX (after the factorisation)
  float* const Gi = sm.ldl.Wb;  // G^-1, row-major, stride KMAX
  __nv_bfloat16* const Vs = KMAX <= 32 ? sm.Vs : reinterpret_cast<__nv_bfloat16*>(sm.ldl.Gs);
  const int b = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool factors = MODE == kSolveSelf || (MODE == kSolveShared && blockIdx.y == 0);
  float* rec = MODE != kSolveSelf ? MD + static_cast<size_t>(b) * ldl_record_floats<KMAX>()
                                  : nullptr;
  unsigned long long* const tr =
      trace ? trace + (blockIdx.y * gridDim.x + blockIdx.x) % kTraceCtas * kTraceSlots : nullptr;
  if (tr && tid == 0) tr[0] = sm100::globaltimer_ns();
  if (!defer_wait) sm100::pdl_wait();
  if (tr && tid == 0) tr[2] = sm100::globaltimer_ns();
  sm100::pdl_launch_dependents();

  const int t0 = blockIdx.y * ROWS;
  const int nrows = min(ROWS, T - t0);
  __nv_bfloat16* const rows = L + (static_cast<size_t>(b) * T + t0) * k;
  // Stage the block's rows (zero beyond k and beyond nrows) in 16-byte pieces
  // (k is a multiple of 8, so every row starts on a 16-byte boundary).
  auto stage_rows = [&](bool async) {
    constexpr int C8 = KMAX / 8;
    for (int e = tid; e < ROWS * C8; e += kLtThreads) {
      const int rr = e / C8, c8 = e % C8;
      const bool valid = rr < nrows && 8 * c8 < k &&
                         sm100::in_bounds(status, (rows - L) + static_cast<size_t>(rr) * k + 8 * c8,
                                          8, static_cast<size_t>(gridDim.x) * T * k);
      const __nv_bfloat16* src = valid ? rows + static_cast<size_t>(rr) * k + 8 * c8 : rows;
      __nv_bfloat16* dst = Vs + rr * VS + 8 * c8;
      if (async)
        sm100::cp_async_16(sm100::smem_u32(dst), src, valid ? 16u : 0u);
      else
        *reinterpret_cast<uint4*>(dst) =
            valid ? __ldcg(reinterpret_cast<const uint4*>(src)) : make_uint4(0, 0, 0, 0);
    }
    if (async) sm100::cp_async_commit();
  };
  if constexpr (KMAX <= 32) {
    stage_rows(true);  // lands while the factorisation runs
  } else {
    // read after the factorisation (the projection wrote them; bring them to L2)
    for (int e = tid; e < nrows; e += kLtThreads)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(rows + static_cast<size_t>(e) * k));
  }

  if (factors) {
    const float* Gb = G + static_cast<size_t>(b) * k * k;
    constexpr int GPT = KMAX * KMAX / kLtThreads;
    float g[GPT];
#pragma unroll
    for (int u = 0; u < GPT; ++u) {  // every load in flight at once
      const int e = tid + u * kLtThreads, i = e / KMAX, q = e % KMAX;
      g[u] = i < k && q < k ? __ldcg(Gb + i * k + q) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < GPT; ++u) {
      const int e = tid + u * kLtThreads, i = e / KMAX, q = e % KMAX;
      sm.ldl.Gs[i * LD + q] =
          i < k && q < k ? g[u] + (i == q ? lambda : 0.f) : (i == q ? 1.f : 0.f);
    }
    __syncthreads();
    if (tr && tid == 0) tr[3] = sm100::globaltimer_ns();
    // M is emitted over ldl.Gs, whose last read precedes the emits
    const bool ok = ldl_blocked<KMAX, kLtThreads>(
        sm.ldl, k, tid, [] { __syncthreads(); },
        [&](int i, int q, float m) { Ma[i * KMAX + q] = m; }, [](int, float) {},
        tr ? tr + 40 : nullptr);
    __syncthreads();
    // G^-1 = M^T D^-1 M, one 16 x 16 block (Q, J) per warp and step: lane
    // (r, h) sums over rows i >= 16 max(Q, J) of M[i][16Q + r] D^-1[i] times
    // M[i][16J + 8h .. +8] (M is zero above its diagonal).
    {
      const int r = lane & 15, h = lane >> 4;
      for (int blk = warp; blk < NB * NB; blk += kLtThreads / 32) {
        const int Q = blk / NB, J = blk % NB;
        float acc[8] = {};
        for (int i = 16 * max(Q, J); i < KMAX; ++i) {
          const float a = Ma[i * KMAX + 16 * Q + r] * sm.ldl.dinv[i];
          const float4 b0 = *reinterpret_cast<const float4*>(&Ma[i * KMAX + 16 * J + 8 * h]);
          const float4 b1 = *reinterpret_cast<const float4*>(&Ma[i * KMAX + 16 * J + 8 * h + 4]);
          acc[0] = fmaf(a, b0.x, acc[0]);
          acc[1] = fmaf(a, b0.y, acc[1]);
          acc[2] = fmaf(a, b0.z, acc[2]);
          acc[3] = fmaf(a, b0.w, acc[3]);
          acc[4] = fmaf(a, b1.x, acc[4]);
          acc[5] = fmaf(a, b1.y, acc[5]);
          acc[6] = fmaf(a, b1.z, acc[6]);
          acc[7] = fmaf(a, b1.w, acc[7]);
        }
        float* dst = &Gi[(16 * Q + r) * KMAX + 16 * J + 8 * h];
        *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
    if (MODE == kSolveShared) {
      __syncthreads();
      for (int e = tid; e < KMAX * KMAX / 4; e += kLtThreads)
        reinterpret_cast<float4*>(rec)[e] = reinterpret_cast<const float4*>(Gi)[e];
      if (tid == 0) rec[KMAX * KMAX] = ok ? 0.f : 1.f;
      // the whole record before the flag: the barrier orders the block's
      // writes before thread 0's fence, whose release covers them
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        sm100::st_release_gpu(flags + b, 1);
      }
    }
  } else {
    if (tid == 0) {
      int bad = 0;
      const unsigned long long deadline = sm100::globaltimer_ns() + sm100::kWaitLimitNs;
      while (sm100::ld_acquire_gpu(flags + b) == 0) {
        if (sm100::globaltimer_ns() > deadline) {
          atomicOr(status, sm100::kStatusTimeout);
          bad = 1;
          break;
        }
        __nanosleep(128);
      }
      sm.ldl.bad = bad;
    }
    __syncthreads();
    // the record: G^-1 (row-major), the failure flag
    for (int e = tid; e < KMAX * KMAX / 4; e += kLtThreads)
      reinterpret_cast<float4*>(Gi)[e] = __ldcg(reinterpret_cast<const float4*>(rec) + e);
    __syncthreads();
    if (tid == 0 && __ldcg(rec + KMAX * KMAX) != 0.f) sm.ldl.bad = 1;
  }
  __syncthreads();  // G^-1 complete; Gs and Mb are free
  if constexpr (KMAX <= 32) {
    sm100::cp_async_wait_all();
  } else {
    stage_rows(false);
  }
  __syncthreads();
  if (tr && tid == 0) tr[4] = sm100::globaltimer_ns();
  const bool zero = sm.ldl.bad != 0;

  // W = V G^-1 over the staged rows, 64 rows per pass: thread tile RT rows x
  // 4 columns (cg: column group, rg: row group), K in steps of 4.
  constexpr int CG = KMAX / 4;
  constexpr int RT = 64 * KMAX / (4 * kLtThreads);
  const int cg = tid % CG, rg = tid / CG;
#pragma unroll 1
  for (int p0 = 0; p0 < nrows; p0 += 64) {
    float acc[RT][4];
#pragma unroll
    for (int rr = 0; rr < RT; ++rr)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[rr][c] = 0.f;
#pragma unroll 4
    for (int i4 = 0; i4 < KMAX / 4; ++i4) {
      float4 gq[4];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
        gq[ii] = *reinterpret_cast<const float4*>(&Gi[(4 * i4 + ii) * KMAX + 4 * cg]);
#pragma unroll
      for (int rr = 0; rr < RT; ++rr) {
        const uint2 vv = *reinterpret_cast<const uint2*>(&Vs[(p0 + RT * rg + rr) * VS + 4 * i4]);
        const float v[4] = {__uint_as_float(vv.x << 16), __uint_as_float(vv.x & 0xffff0000u),
                            __uint_as_float(vv.y << 16), __uint_as_float(vv.y & 0xffff0000u)};
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
          acc[rr][0] = fmaf(v[ii], gq[ii].x, acc[rr][0]);
          acc[rr][1] = fmaf(v[ii], gq[ii].y, acc[rr][1]);
          acc[rr][2] = fmaf(v[ii], gq[ii].z, acc[rr][2]);
          acc[rr][3] = fmaf(v[ii], gq[ii].w, acc[rr][3]);
        }
      }
    }
#pragma unroll
    for (int rr = 0; rr < RT; ++rr) {
      const int rl = p0 + RT * rg + rr;
      if (rl >= nrows || 4 * cg >= k) continue;
      __nv_bfloat16* dst = rows + static_cast<size_t>(rl) * k + 4 * cg;
      if (!sm100::in_bounds(status, dst - L, 4, static_cast<size_t>(gridDim.x) * T * k)) continue;
      // a failed factorisation writes zeros (not alpha times a non-finite value)
      const __nv_bfloat162 lo = __floats2bfloat162_rn(zero ? 0.f : alpha * acc[rr][0],
                                                      zero ? 0.f : alpha * acc[rr][1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(zero ? 0.f : alpha * acc[rr][2],
                                                      zero ? 0.f : alpha * acc[rr][3]);
      uint2 w;
      w.x = *reinterpret_cast<const uint32_t*>(&lo);
      w.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(dst) = w;
      if (Llo != nullptr) {  // the rounding errors of the four values just stored
        const float2 l2 = __bfloat1622float2(lo), h2 = __bfloat1622float2(hi);
        const __nv_bfloat162 elo = __floats2bfloat162_rn(zero ? 0.f : alpha * acc[rr][0] - l2.x,
                                                         zero ? 0.f : alpha * acc[rr][1] - l2.y);
        const __nv_bfloat162 ehi = __floats2bfloat162_rn(zero ? 0.f : alpha * acc[rr][2] - h2.x,
                                                         zero ? 0.f : alpha * acc[rr][3] - h2.y);
        uint2 we;
        we.x = *reinterpret_cast<const uint32_t*>(&elo);
        we.y = *reinterpret_cast<const uint32_t*>(&ehi);
        *reinterpret_cast<uint2*>(Llo + (dst - L)) = we;
      }
    }
  }
  if (tr && tid == 0) tr[5] = sm100::globaltimer_ns();
  if (tid == 0 && blockIdx.y == 0 && zero) atomicOr(status, sm100::kStatusPivot);
  if (defer_wait) sm100::pdl_wait();
  if (tr && tid == 0) tr[8] = sm100::globaltimer_ns();
}

// Newton-Schulz inverse of G_b + lambda I, one CTA per instance ([DyRA]
// Sec. 2.4 names a Newton-Schulz iterative solver for larger correction ranks
// in place of the sequential Cholesky solve). From X_0 = I / ||G||_inf, whose
// spectrum lies in (0, 1], the iteration X <- X (2 I - G X) squares the
// residual I - G X at every step; it stops when the largest entry of the
// residual is below 1e-6, when it stops shrinking near the fp32 rounding
// floor, or after max_iters steps. The result is published as the solve's
// factor record of the instance (G_b^-1 row-major with stride KMAX, then a
// failure flag) behind its ready flag, which the kSolveGiven solve reads. A
// residual that is not finite, or is not below 1e-2 at the end, flags the
// instance: its correction becomes zero and DYRA_STATUS_NONPOSITIVE_PIVOT is
// raised.
constexpr int kNsThreads = 256;
template <int KMAX>
__host__ __device__ constexpr int ns_ld() {
  return KMAX + 4;  // row stride of the kernel's three KMAX x KMAX tiles
}
template <int KMAX>
constexpr size_t ns_smem_bytes() {
  return 3 * sizeof(float) * KMAX * ns_ld<KMAX>();
}

template <int KMAX>
__global__ void __launch_bounds__(kNsThreads)
    ns_inverse_kernel(const float* __restrict__ G, int k, float lambda, int max_iters, float* MD,
                      int* flags, int* status) {
  constexpr int LD = ns_ld<KMAX>();
  constexpr int TPR = KMAX / 16;  // each thread owns a TPR x TPR block of the product
  extern __shared__ __align__(16) float ns_smem[];
  float* const Gs = ns_smem;          // G + lambda I, zero beyond k
  float* const Xs = Gs + KMAX * LD;   // the iterate X
  float* const Ps = Xs + KMAX * LD;   // G X
  __shared__ float red[kNsThreads / 32];
  __shared__ float resid;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int ti = tid / 16, tj = tid % 16;  // thread block row / column
  sm100::pdl_launch_dependents();
  const float* Gb = G + static_cast<size_t>(b) * k * k;
  for (int e = tid; e < KMAX * KMAX; e += kNsThreads) {
    const int i = e / KMAX, q = e % KMAX;
    Gs[i * LD + q] = i < k && q < k ? __ldcg(Gb + i * k + q) + (i == q ? lambda : 0.f) : 0.f;
  }
  __syncthreads();
  // ||G||_inf: the largest absolute row sum
  float rs = 0.f;
  if (tid < k)
    for (int q = 0; q < k; ++q) rs += fabsf(Gs[tid * LD + q]);
  for (int o = 16; o > 0; o >>= 1) rs = fmaxf(rs, __shfl_xor_sync(0xffffffffu, rs, o));
  if ((tid & 31) == 0) red[tid >> 5] = rs;
  __syncthreads();
  float gnorm = 0.f;
  for (int w = 0; w < kNsThreads / 32; ++w) gnorm = fmaxf(gnorm, red[w]);
  const float x0 = gnorm > 0.f && isfinite(gnorm) ? 1.f / gnorm : 0.f;
  for (int e = tid; e < KMAX * KMAX; e += kNsThreads) {
    const int i = e / KMAX, q = e % KMAX;
    Xs[i * LD + q] = i == q && i < k ? x0 : 0.f;
  }
  __syncthreads();
  // C = A B for the thread's block (rows TPR*ti.., columns TPR*tj..)
  auto block_product = [&](const float* A, const float* Bm, float (&c)[TPR][TPR]) {
#pragma unroll
    for (int u = 0; u < TPR; ++u)
#pragma unroll
      for (int v = 0; v < TPR; ++v) c[u][v] = 0.f;
    for (int q = 0; q < k; ++q) {
      float a[TPR], bv[TPR];
#pragma unroll
      for (int u = 0; u < TPR; ++u) a[u] = A[(TPR * ti + u) * LD + q];
#pragma unroll
      for (int v = 0; v < TPR; ++v) bv[v] = Bm[q * LD + TPR * tj + v];
#pragma unroll
      for (int u = 0; u < TPR; ++u)
#pragma unroll
        for (int v = 0; v < TPR; ++v) c[u][v] = fmaf(a[u], bv[v], c[u][v]);
    }
  };
  float prev = 3.4e38f, r = 3.4e38f;
  for (int it = 0; it < max_iters; ++it) {
    float c[TPR][TPR];
    block_product(Gs, Xs, c);  // P = G X
    float mx = 0.f;
#pragma unroll
    for (int u = 0; u < TPR; ++u)
#pragma unroll
      for (int v = 0; v < TPR; ++v) {
        const int i = TPR * ti + u, q = TPR * tj + v;
        Ps[i * LD + q] = c[u][v];
        if (i < k && q < k) {
          const float d = (i == q ? 1.f : 0.f) - c[u][v];
          mx = isfinite(d) ? fmaxf(mx, fabsf(d)) : 3.4e38f;
        }
      }
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    if (tid == 0) {
      float m = 0.f;
      for (int w = 0; w < kNsThreads / 32; ++w) m = fmaxf(m, red[w]);
      resid = m;
    }
    __syncthreads();
    r = resid;
    if (r < 1e-6f || (r < 1e-2f && r > 0.5f * prev)) break;
    prev = r;
    block_product(Xs, Ps, c);  // X P
    __syncthreads();           // every read of X done
#pragma unroll
    for (int u = 0; u < TPR; ++u)
#pragma unroll
      for (int v = 0; v < TPR; ++v) {
        const int i = TPR * ti + u, q = TPR * tj + v;
        Xs[i * LD + q] = 2.f * Xs[i * LD + q] - c[u][v];
      }
    __syncthreads();
  }
  const bool bad = !(r < 1e-2f);
  float* rec = MD + static_cast<size_t>(b) * ldl_record_floats<KMAX>();
  const size_t rec_extent = static_cast<size_t>(gridDim.x) * ldl_record_floats<KMAX>();
  for (int e = tid; e < KMAX * KMAX; e += kNsThreads) {
    const int i = e / KMAX, q = e % KMAX;
    if (sm100::in_bounds(status, (rec - MD) + e, 1, rec_extent)) rec[e] = Xs[i * LD + q];
  }
  if (tid == 0) rec[KMAX * KMAX] = bad ? 1.f : 0.f;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    sm100::st_release_gpu(flags + b, 1);
    if (bad) atomicOr(status, sm100::kStatusPivot);
  }
  // the grid before this one (the GEMM for Q) is complete before this one
  // is, so the stages after the solve may rely on both
  sm100::pdl_wait();
}

// General variant of the same (any k <= 128): every CTA factors G_b itself
// (Cholesky G_b = R R^T in shared memory) and solves R R^T w = l for 128 rows
// of L_b, one per thread.
__global__ void __launch_bounds__(kSolveThreads)
    ltilde_general_kernel(const float* __restrict__ G, __nv_bfloat16* L, __nv_bfloat16* Llo, int T,
                          int k, float lambda, float alpha, int* status, int defer_wait) {
  extern __shared__ float sm[];
  const int ldg = k + 1;
  float* R = sm;                // k x (k+1): lower triangle becomes R
  float* Ycol = sm + k * ldg;   // k x 128: one row of L_b per thread
  __shared__ int bad;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  if (!defer_wait) sm100::pdl_wait();
  sm100::pdl_launch_dependents();
  if (tid == 0) bad = 0;
  const float* Gb = G + static_cast<size_t>(b) * k * k;
  for (int idx = tid; idx < k * k; idx += kSolveThreads) {
    const int i = idx / k, i2 = idx - (idx / k) * k;
    R[i * ldg + i2] = Gb[idx] + (i == i2 ? lambda : 0.f);
  }
  __syncthreads();
  for (int j = 0; j < k; ++j) {
    if (tid == 0) {
      const float d = R[j * ldg + j];
      if (!(d > 0.f) || !isfinite(d)) {
        bad = 1;
        R[j * ldg + j] = 1.f;
      } else {
        R[j * ldg + j] = sqrtf(d);
      }
    }
    __syncthreads();
    const float inv = 1.f / R[j * ldg + j];
    for (int i = j + 1 + tid; i < k; i += kSolveThreads) R[i * ldg + j] *= inv;
    __syncthreads();
    const int m = k - j - 1;
    for (int idx = tid; idx < m * m; idx += kSolveThreads) {
      const int i = j + 1 + idx / m, i2 = j + 1 + (idx - (idx / m) * m);
      if (i2 <= i) R[i * ldg + i2] -= R[i * ldg + j] * R[i2 * ldg + j];
    }
    __syncthreads();
  }
  const int t = blockIdx.y * kSolveThreads + tid;
  if (t < T && sm100::in_bounds(status, (static_cast<size_t>(b) * T + t) * k, k,
                                static_cast<size_t>(gridDim.x) * T * k)) {
    __nv_bfloat16* row = L + (static_cast<size_t>(b) * T + t) * k;
    for (int i = 0; i < k; ++i) Ycol[i * kSolveThreads + tid] = __bfloat162float(row[i]);
    for (int i = 0; i < k; ++i) {  // R y = l
      float acc = Ycol[i * kSolveThreads + tid];
      for (int q = 0; q < i; ++q) acc -= R[i * ldg + q] * Ycol[q * kSolveThreads + tid];
      Ycol[i * kSolveThreads + tid] = acc / R[i * ldg + i];
    }
    for (int i = k - 1; i >= 0; --i) {  // R^T w = y
      float acc = Ycol[i * kSolveThreads + tid];
      for (int q = i + 1; q < k; ++q) acc -= R[q * ldg + i] * Ycol[q * kSolveThreads + tid];
      Ycol[i * kSolveThreads + tid] = acc / R[i * ldg + i];
    }
    const bool zero = bad != 0;
    for (int i = 0; i < k; ++i) {
      const float v = zero ? 0.f : alpha * Ycol[i * kSolveThreads + tid];
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      row[i] = h;
      if (Llo != nullptr) Llo[(row - L) + i] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
  if (tid == 0 && blockIdx.y == 0 && bad) atomicOr(status, sm100::kStatusPivot);
  if (defer_wait) sm100::pdl_wait();
}

// C[b][m][n] (+)= alpha sum_q A[b][m][q] * Bm[b][q][n] (+ bias[n]) with
// arbitrary element strides.
// kGK: the k step. Long K takes 64 (64 x 64 elements of each operand in
// flight per step, a quarter of the dependent load round trips of 16); short
// K takes 16, which wastes less work on the zero-filled tail.
constexpr int kGT = 64;   // tile
template <typename TA, typename TB, typename TC, int kGK>
__global__ void __launch_bounds__(256)
    simt_gemm_kernel(int M, int N, int K, const TA* __restrict__ A, int64_t am, int64_t ak,
                     int64_t ab, const TB* __restrict__ Bm, int64_t bk, int64_t bn, int64_t bb,
                     TC* __restrict__ C, int64_t cm, int64_t cn, int64_t cb, int accumulate,
                     float alpha, const TC* __restrict__ bias, int64_t bias_b) {
  __shared__ float As[kGK][kGT + 1];
  __shared__ float Bs[kGK][kGT + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * kGT, n0 = blockIdx.x * kGT;
  const int64_t batch = blockIdx.z;
  A += batch * ab;
  Bm += batch * bb;
  C += batch * cb;
  // consecutive threads walk the operand's unit-stride dimension (coalesced)
  const bool a_k_fast = ak == 1, b_k_fast = bk == 1 && bn != 1;
  float acc[4][4] = {};
  constexpr int kPer = kGK * kGT / 256;  // elements of each operand per thread and step
  for (int q0 = 0; q0 < K; q0 += kGK) {
    // every load of the step in flight before the first store to shared memory
    float va[kPer], vb[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int idx = threadIdx.x + 256 * j;
      const int qa = a_k_fast ? idx % kGK : idx / kGT, ma = a_k_fast ? idx / kGK : idx % kGT;
      const int gm = m0 + ma, gqa = q0 + qa;
      va[j] = (gm < M && gqa < K) ? to_f<TA>(A[gm * am + gqa * ak]) : 0.f;
      const int qb = b_k_fast ? idx % kGK : idx / kGT, nb = b_k_fast ? idx / kGK : idx % kGT;
      const int gn = n0 + nb, gqb = q0 + qb;
      vb[j] = (gn < N && gqb < K) ? to_f<TB>(Bm[gqb * bk + gn * bn]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int idx = threadIdx.x + 256 * j;
      const int qa = a_k_fast ? idx % kGK : idx / kGT, ma = a_k_fast ? idx / kGK : idx % kGT;
      const int qb = b_k_fast ? idx % kGK : idx / kGT, nb = b_k_fast ? idx / kGK : idx % kGT;
      As[qa][ma] = va[j];
      Bs[qb][nb] = vb[j];
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
      float v = alpha * acc[i][j];
      if (bias) v += to_f<TC>(bias[batch * bias_b + gn]);
      if (accumulate) v += to_f<TC>(*dst);
      *dst = from_f<TC>(v);
    }
  }
}

template <typename TA, typename TB, typename TC>
int gemm(int M, int N, int K, const TA* A, int64_t am, int64_t ak, int64_t ab, const TB* Bm,
         int64_t bk, int64_t bn, int64_t bb, TC* C, int64_t cm, int64_t cn, int64_t cb,
         int batches, int accumulate, cudaStream_t s, float alpha = 1.f,
         const TC* bias = nullptr, int64_t bias_b = 0) {
  if (M <= 0 || N <= 0 || batches <= 0) return 0;
  dim3 grid((N + kGT - 1) / kGT, (M + kGT - 1) / kGT, batches);
  if (K >= 128)
    simt_gemm_kernel<TA, TB, TC, 64><<<grid, 256, 0, s>>>(M, N, K, A, am, ak, ab, Bm, bk, bn, bb,
                                                          C, cm, cn, cb, accumulate, alpha, bias,
                                                          bias_b);
  else
    simt_gemm_kernel<TA, TB, TC, 16><<<grid, 256, 0, s>>>(M, N, K, A, am, ak, ab, Bm, bk, bn, bb,
                                                          C, cm, cn, cb, accumulate, alpha, bias,
                                                          bias_b);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// out[row][q * P + p] = in[row][p * Q + q] for every row (p < P, q < Q): each
// row, read as a row-major P x Q grid, is written back transposed. This is the
// perfect shuffle of the Monarch factorisation ([DyRA] App. B), and the block
// transpose of its factors. A block stages one row in shared memory at a time
// (16-byte loads); the stores are 16-byte when P is a multiple of 8.
constexpr int kShuffleThreads = 256;

__global__ void __launch_bounds__(kShuffleThreads)
    grid_transpose_kernel(const __nv_bfloat16* __restrict__ in, __nv_bfloat16* __restrict__ out,
                          int64_t rows, int P, int Q) {
  extern __shared__ __align__(16) __nv_bfloat16 row_s[];
  const int n = P * Q;  // a multiple of 8
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const __nv_bfloat16* src = in + row * n;
    __nv_bfloat16* dst = out + row * n;
    for (int e = 8 * threadIdx.x; e < n; e += 8 * kShuffleThreads)
      *reinterpret_cast<uint4*>(row_s + e) = __ldg(reinterpret_cast<const uint4*>(src + e));
    __syncthreads();
    if (P % 8 == 0) {
      for (int o = 8 * threadIdx.x; o < n; o += 8 * kShuffleThreads) {
        const int q = o / P, p = o - q * P;  // outputs o .. o + 7 share q
        __align__(16) __nv_bfloat16 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = row_s[(p + u) * Q + q];
        *reinterpret_cast<uint4*>(dst + o) = *reinterpret_cast<const uint4*>(v);
      }
    } else {
      for (int o = threadIdx.x; o < n; o += kShuffleThreads) {
        const int q = o / P, p = o - q * P;
        dst[o] = row_s[p * Q + q];
      }
    }
    __syncthreads();
  }
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

template <typename TOut, int KMAX>
int launch_solve_ldl(cudaLaunchConfig_t& cfg, const float* TG, int splits, int64_t B, int k,
                     int d_in, float lambda, TOut* Tp, int* status, unsigned long long* trace,
                     float alpha) {
  auto kfn = solve_ldl_kernel<TOut, KMAX>;
  static KernelSetup setup;
  const int d = setup_device();
  if (d < 0) return -1;
  if (setup.smem[d].load() == 0) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sizeof(SolveSmem<KMAX>))) != cudaSuccess ||
        cudaFuncSetAttribute(kfn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
            cudaSuccess)
      return -1;
    setup.smem[d].store(static_cast<uint32_t>(sizeof(SolveSmem<KMAX>)));
  }
  cfg.gridDim = dim3(static_cast<unsigned>(B),
                     static_cast<unsigned>((d_in + kSolveCols - 1) / kSolveCols));
  cfg.blockDim = dim3(kSolveThreads2);
  cfg.dynamicSmemBytes = sizeof(SolveSmem<KMAX>);
  return cudaLaunchKernelEx(&cfg, kfn, TG, splits, static_cast<int>(B), k, d_in, lambda, Tp,
                            status, trace, alpha) == cudaSuccess
             ? 0
             : -1;
}

template <typename TOut>
int launch_solve(const float* TG, int splits, int64_t B, int k, int d_in, float lambda, TOut* Tp,
                 int* status, cudaStream_t s, bool pdl, unsigned long long* trace, float alpha) {
  if (B == 0 || k == 0) return 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cfg.stream = s;
  if (k <= 32)
    return launch_solve_ldl<TOut, 32>(cfg, TG, splits, B, k, d_in, lambda, Tp, status, trace,
                                      alpha);
  if (k <= 64)
    return launch_solve_ldl<TOut, 64>(cfg, TG, splits, B, k, d_in, lambda, Tp, status, trace,
                                      alpha);
  const size_t smem = (static_cast<size_t>(k) * (k + 1) + static_cast<size_t>(k) * kSolveThreads) *
                      sizeof(float);
  auto kfn = solve_kernel<TOut>;
  static KernelSetup setup;
  const int d = setup_device();
  if (d < 0) return -1;
  if (smem > 48 * 1024 && smem > setup.smem[d].load()) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -1;
    setup.smem[d].store(static_cast<uint32_t>(smem));
  }
  cfg.gridDim = dim3(static_cast<unsigned>(B), static_cast<unsigned>((d_in + kSolveThreads - 1) / kSolveThreads));
  cfg.blockDim = dim3(kSolveThreads);
  cfg.dynamicSmemBytes = smem;
  return cudaLaunchKernelEx(&cfg, kfn, TG, splits, static_cast<int>(B), k, d_in, lambda, Tp,
                            status, alpha) == cudaSuccess
             ? 0
             : -1;
}

int ltilde_rows_per_block(int k) {
  return k <= 32 ? lt_rows<32>() : k <= 64 ? lt_rows<64>() : kSolveThreads;
}

size_t ltilde_smem_bytes(int k) {
  if (k <= 0) return 0;
  if (k <= 32) return sizeof(LtSmem<32>);
  if (k <= 64) return sizeof(LtSmem<64>);
  return (static_cast<size_t>(k) * (k + 1) + static_cast<size_t>(k) * kSolveThreads) * sizeof(float);
}

template <int KMAX, int MODE>
int launch_ltilde_fast(cudaLaunchConfig_t& cfg, const float* G, __nv_bfloat16* L,
                       __nv_bfloat16* Llo, float* MD, int* flags, int64_t B, int64_t T, int k,
                       float lambda, float alpha, int* status, int defer_wait,
                       unsigned long long* trace) {
  auto kfn = ltilde_kernel<KMAX, MODE>;
  static KernelSetup setup;
  const int d = setup_device();
  if (d < 0) return -1;
  if (setup.smem[d].load() == 0) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sizeof(LtSmem<KMAX>))) != cudaSuccess ||
        cudaFuncSetAttribute(kfn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
            cudaSuccess)
      return -1;
    setup.smem[d].store(static_cast<uint32_t>(sizeof(LtSmem<KMAX>)));
  }
  // blockIdx.x = instance, blockIdx.y = chunk of rows: the chunk-0 CTAs (the
  // factoring ones in the shared mode) are the grid's first B CTAs.
  cfg.gridDim = dim3(static_cast<unsigned>(B),
                     static_cast<unsigned>((T + lt_rows<KMAX>() - 1) / lt_rows<KMAX>()));
  cfg.blockDim = dim3(kLtThreads);
  cfg.dynamicSmemBytes = sizeof(LtSmem<KMAX>);
  return cudaLaunchKernelEx(&cfg, kfn, G, L, Llo, MD, flags, static_cast<int>(T), k, lambda, alpha,
                            status, defer_wait, trace) == cudaSuccess
             ? 0
             : -1;
}

int launch_ns_inverse(const float* G, int64_t B, int k, float lambda, int max_iters, float* MD,
                      int* flags, int* status, cudaStream_t s) {
  if (B == 0 || k == 0) return 0;
  if (k > 64 || MD == nullptr || flags == nullptr || B > 2147483647) return -1;
  static KernelSetup setup;
  const int d = setup_device();
  if (d < 0) return -1;
  if (setup.smem[d].load() == 0) {
    if (cudaFuncSetAttribute(ns_inverse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(ns_smem_bytes<64>())) != cudaSuccess)
      return -1;
    setup.smem[d].store(static_cast<uint32_t>(ns_smem_bytes<64>()));
  }
  if (k <= 32)
    ns_inverse_kernel<32><<<static_cast<unsigned>(B), kNsThreads, ns_smem_bytes<32>(), s>>>(
        G, k, lambda, max_iters, MD, flags, status);
  else
    ns_inverse_kernel<64><<<static_cast<unsigned>(B), kNsThreads, ns_smem_bytes<64>(), s>>>(
        G, k, lambda, max_iters, MD, flags, status);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_ltilde(const float* G, void* L, void* Llo, float* MD, int* flags, int mode, int64_t B,
                  int64_t T, int k, float lambda, float alpha, int* status, cudaStream_t s, bool pdl,
                  bool defer_wait, unsigned long long* trace) {
  const int dw = pdl && defer_wait ? 1 : 0;
  if (B == 0 || T == 0 || k == 0) return 0;
  if (k % 8 != 0) return -1;  // bf16 plans: 16-byte rows of L
  if (mode != kSolveSelf && (MD == nullptr || flags == nullptr || k > 64)) return -1;
  if ((T + ltilde_rows_per_block(k) - 1) / ltilde_rows_per_block(k) > 65535 || B > 2147483647)
    return -1;
  auto* Lb = static_cast<__nv_bfloat16*>(L);
  auto* Lo = static_cast<__nv_bfloat16*>(Llo);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cfg.stream = s;
  if (k <= 32)
    return mode == kSolveShared
               ? launch_ltilde_fast<32, kSolveShared>(cfg, G, Lb, Lo, MD, flags, B, T, k, lambda,
                                                      alpha, status, dw, trace)
           : mode == kSolveGiven
               ? launch_ltilde_fast<32, kSolveGiven>(cfg, G, Lb, Lo, MD, flags, B, T, k, lambda,
                                                     alpha, status, dw, trace)
               : launch_ltilde_fast<32, kSolveSelf>(cfg, G, Lb, Lo, MD, flags, B, T, k, lambda,
                                                    alpha, status, dw, trace);
  if (k <= 64)
    return mode == kSolveShared
               ? launch_ltilde_fast<64, kSolveShared>(cfg, G, Lb, Lo, MD, flags, B, T, k, lambda,
                                                      alpha, status, dw, trace)
           : mode == kSolveGiven
               ? launch_ltilde_fast<64, kSolveGiven>(cfg, G, Lb, Lo, MD, flags, B, T, k, lambda,
                                                     alpha, status, dw, trace)
               : launch_ltilde_fast<64, kSolveSelf>(cfg, G, Lb, Lo, MD, flags, B, T, k, lambda,
                                                    alpha, status, dw, trace);
  const size_t smem = ltilde_smem_bytes(k);
  static KernelSetup setup;
  const int d = setup_device();
  if (d < 0) return -1;
  if (smem > 48 * 1024 && smem > setup.smem[d].load()) {
    if (cudaFuncSetAttribute(ltilde_general_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -1;
    setup.smem[d].store(static_cast<uint32_t>(smem));
  }
  if ((T + kSolveThreads - 1) / kSolveThreads > 65535) return -1;
  cfg.gridDim = dim3(static_cast<unsigned>(B),
                     static_cast<unsigned>((T + kSolveThreads - 1) / kSolveThreads));
  cfg.blockDim = dim3(kSolveThreads);
  cfg.dynamicSmemBytes = smem;
  return cudaLaunchKernelEx(&cfg, ltilde_general_kernel, G, Lb, Lo, static_cast<int>(T), k, lambda,
                            alpha, status, dw) == cudaSuccess
             ? 0
             : -1;
}

template int launch_solve<float>(const float*, int, int64_t, int, int, float, float*, int*,
                                 cudaStream_t, bool, unsigned long long*, float);
template int launch_solve<__nv_bfloat16>(const float*, int, int64_t, int, int, float,
                                         __nv_bfloat16*, int*, cudaStream_t, bool,
                                         unsigned long long*, float);

int launch_grid_transpose(const void* in, void* out, int64_t rows, int P, int Q, int sm_count,
                          cudaStream_t s) {
  if (rows == 0) return 0;
  const int64_t n = static_cast<int64_t>(P) * Q;
  if (P < 1 || Q < 1 || n % 8 != 0 || n > 49152) return -1;
  const size_t smem = static_cast<size_t>(n) * sizeof(__nv_bfloat16);
  static KernelSetup setup;
  const int d = setup_device();
  if (d < 0) return -1;
  if (smem > 48 * 1024 && smem > setup.smem[d].load()) {
    if (cudaFuncSetAttribute(grid_transpose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -1;
    setup.smem[d].store(static_cast<uint32_t>(smem));
  }
  const int64_t blocks = std::min<int64_t>(rows, static_cast<int64_t>(std::max(sm_count, 1)) * 8);
  grid_transpose_kernel<<<static_cast<unsigned>(blocks), kShuffleThreads, smem, s>>>(
      static_cast<const __nv_bfloat16*>(in), static_cast<__nv_bfloat16*>(out), rows, P, Q);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

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
// strided batched SIMT GEMM, with fp32 storage of every intermediate. With
// more than two half-steps, further L and R updates follow Alg. 1's pair
// ([DyRA] Sec. 2.2, Eq. 4-5 with the ridge of footnote 2; Sec. 3.3):
//   L update  L_b = X_b (R_b W_res)^T (R_b R_b^T + lambda I)^-1
//   R update  R_b = (L_b^T L_b + lambda I)^-1 (L_b^T X_b) W_res^T
// and the output takes the last pair. Both updates go through the same ridge
// solve: the R update solves for R_b from [L_b^T X_b | L_b^T L_b], the L
// update for L_b^T from [(X_b (R_b W_res)^T)^T | R_b R_b^T].
template <typename T>
int launch_simt_forward(const SimtForward<T>& a, const DeviceInfo&, cudaStream_t s) {
  const int64_t N = a.B * a.Trows;
  if (N == 0) return 0;
  const int rk = a.r + a.k;
  const int k = a.weight_only ? 0 : a.k;
  const int Bn = static_cast<int>(a.B);
  const int Tr = static_cast<int>(a.Trows);
  const int steps = k > 0 ? a.half_steps : 0;
  if (k > 0 && (steps < 2 || (steps > 2 && (!a.Lt || !a.P2 || !a.TG2)))) return -1;
  // [Z | L] = X [V | P]
  if (gemm(static_cast<int>(N), rk, a.d_in, a.X, a.d_in, 1, 0, a.VPt, 1, a.d_in, 0, a.ZL, rk, 1,
           0, 1, 0, s))
    return -1;
  // the current L_b: element (t, i) at Lp[b * lb + t * lm + i * lq]
  const T* Lp = a.ZL + a.r;
  int64_t lm = rk, lq = 1, lb = static_cast<int64_t>(Tr) * rk;
  for (int h = 1; h < steps; ++h) {
    if (h % 2 == 1) {  // R update from the current L
      const int J = a.d_in + k;
      // T_b = L_b^T X_b  -> TG[b][i][j], j < d_in
      if (gemm(k, a.d_in, Tr, Lp, lq, lm, lb, a.X, a.d_in, 1, static_cast<int64_t>(Tr) * a.d_in,
               a.TG, J, 1, static_cast<int64_t>(k) * J, Bn, 0, s))
        return -1;
      // G_b = L_b^T L_b -> TG[b][i][d_in + i']
      if (gemm(k, k, Tr, Lp, lq, lm, lb, Lp, lm, lq, lb, a.TG + a.d_in, J, 1,
               static_cast<int64_t>(k) * J, Bn, 0, s))
        return -1;
      if (launch_solve<T>(a.TG, 1, a.B, k, a.d_in, a.lambda, a.Tp, a.status, s, false, nullptr,
                          1.f))
        return -1;
      // R = T' W_res^T  (B*k x d_out)
      if (gemm(Bn * k, a.d_out, a.d_in, a.Tp, a.d_in, 1, 0, a.W_res, 1, a.d_in, 0, a.Cm, a.d_out,
               1, 0, 1, 0, s))
        return -1;
    } else {  // L update from the current R (in Cm)
      const int J = Tr + k;
      // P2 = R W_res  (B*k x d_in)
      if (gemm(Bn * k, a.d_in, a.d_out, a.Cm, a.d_out, 1, 0, a.W_res, a.d_in, 1, 0, a.P2, a.d_in,
               1, 0, 1, 0, s))
        return -1;
      // (X_b P2_b^T)^T -> TG2[b][i][t], t < Tr
      if (gemm(k, Tr, a.d_in, a.P2, a.d_in, 1, static_cast<int64_t>(k) * a.d_in, a.X, 1, a.d_in,
               static_cast<int64_t>(Tr) * a.d_in, a.TG2, J, 1, static_cast<int64_t>(k) * J, Bn, 0,
               s))
        return -1;
      // R_b R_b^T -> TG2[b][i][Tr + i']
      if (gemm(k, k, a.d_out, a.Cm, a.d_out, 1, static_cast<int64_t>(k) * a.d_out, a.Cm, 1,
               a.d_out, static_cast<int64_t>(k) * a.d_out, a.TG2 + Tr, J, 1,
               static_cast<int64_t>(k) * J, Bn, 0, s))
        return -1;
      // L_b^T = (R_b R_b^T + lambda I)^-1 (X_b P2_b^T)^T  -> Lt[b*k + i][t]
      if (launch_solve<T>(a.TG2, 1, a.B, k, Tr, a.lambda, a.Lt, a.status, s, false, nullptr,
                          1.f))
        return -1;
      Lp = a.Lt;
      lm = 1;
      lq = Tr;
      lb = static_cast<int64_t>(k) * Tr;
    }
  }
  if (a.Lblk != nullptr) {
    // Monarch static part: y[j1*b2' + i2] = sum_{m1, j2} x[m1*b2 + j2] L_j2[m1][j1] R_j1[j2][i2],
    // as two strided batched products through Mtmp[row][j2*b1' + j1]
    const int b1 = a.mb1, b2 = a.mb2, b1o = a.mb1o, b2o = a.mb2o;
    const int nmid = b2 * b1o;
    if (gemm(static_cast<int>(N), b1o, b1, a.X, a.d_in, b2, 1, a.Lblk, b1o, 1,
             static_cast<int64_t>(b1) * b1o, a.Mtmp, nmid, 1, b1o, b2, 0, s))
      return -1;
    if (gemm(static_cast<int>(N), b2o, b2, a.Mtmp, nmid, b1o, 1, a.Rblk, b2o, 1,
             static_cast<int64_t>(b2) * b2o, a.Y, a.d_out, 1, b2o, b1o, 0, s, 1.f, a.bias, b2o))
      return -1;
  } else if (gemm(static_cast<int>(N), a.d_out, a.r, a.ZL, rk, 1, 0, a.U, 1, a.r, 0, a.Y, a.d_out,
                  1, 0, 1, 0, s, 1.f, a.bias)) {  // Y = Z U^T (+ b)
    return -1;
  }
  if (k > 0) {
    // Y_b += alpha L_b R_b (the last pair)
    if (gemm(Tr, a.d_out, k, Lp, lm, lq, lb, a.Cm, a.d_out, 1, static_cast<int64_t>(k) * a.d_out,
             a.Y, a.d_out, 1, static_cast<int64_t>(Tr) * a.d_out, Bn, 1, s, a.alpha))
      return -1;
  }
  return 0;
}

template int launch_simt_forward<float>(const SimtForward<float>&, const DeviceInfo&,
                                        cudaStream_t);
template int launch_simt_forward<__nv_bfloat16>(const SimtForward<__nv_bfloat16>&,
                                                const DeviceInfo&, cudaStream_t);

}  // namespace dyra
