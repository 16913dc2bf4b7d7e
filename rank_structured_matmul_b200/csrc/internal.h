// internal.h - interfaces between the C ABI (dyra_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

namespace dyra {

// Launch set-up of one kernel, per device: cudaFuncSetAttribute acts on the
// current device only, so each device of a process is configured on its own
// (plans on several devices may share the process and run from several host
// threads; setting an attribute twice is harmless).
constexpr int kMaxDevices = 64;
struct KernelSetup {
  std::atomic<uint32_t> smem[kMaxDevices];  // dynamic shared memory configured so far
  std::atomic<int> occupancy[kMaxDevices];  // cached occupancy figure (e.g. resident pairs)
};

// The current device, or -1 if it cannot be read or is beyond kMaxDevices.
inline int setup_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return d < kMaxDevices ? d : -1;
}

struct DeviceInfo {
  int device = 0;
  int sm_count = 0;
  int max_smem_optin = 0;
  int smem_per_sm = 0;    // shared memory of one SM, shared by its resident blocks
  int smem_reserved = 0;  // shared memory the system reserves per resident block
  int cc_major = 0, cc_minor = 0;
};

// ---------------------------------------------------------------- TMA ----

// Encode a 2-D or 3-D bf16 tiled tensor map (dims and box innermost first,
// strides in bytes for dims 1..rank-1). swizzle_bytes: 0, 32, 64 or 128.
// Returns false if the driver rejects it.
bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

// --------------------------------------------------- bf16 forward (tcgen05) ----

struct Bf16Forward {
  int d_in, d_out, r, k;
  int64_t B, T;          // instances x rows per instance
  const void* X;         // N x d_in
  void* Y;               // N x d_out
  const void* VPt;       // (r+k) x d_in   ([V | P] transposed)
  const void* U;         // d_out x r
  const void* W_res;     // d_out x d_in
  float lambda;
  bool weight_only;      // skip the correction (k treated as 0)
  // workspace
  void* Z;               // N x r
  void* L;               // N x k
  float* TG;             // B x k x k: G_b (fp32, without the ridge)
  void* Tp;              // (B*k) x d_in: T[b*k + i][j] = (L_b^T X_b)[i][j] (bf16)
  void* Ct;              // d_out x (B*k)
  float* MD;             // B factor records (factor_record_floats(k) floats each), or nullptr
  int* counters;         // B ints: the solve's per-instance flags; cleared by the projection
  int factor_mode;       // who factors G_b: -1 chosen by size, 0 every solve block, 1 the first
  int splits;            // row splits of the Gram reduction
  int split_rows;        // rows per split (multiple of 64)
  int* status;
  cudaEvent_t* stage_events;  // optional: 6 events recorded around the 5 stages
  unsigned long long* trace;  // optional: 5 stages x kTraceCtas x kTraceSlots timestamps
  bool use_pairs;             // run the output stage on CTA pairs
  int proj_pair_min_tiles;    // see proj_shape (0: default)
  int proj_bn = 0;            // projection column tile 128, 192 or 256 (0: proj_shape's choice)
  const void* bias = nullptr;  // d_out bf16 values added to Y, or nullptr
  float alpha = 1.f;           // weight of the correction (the solve scales L~ by it)
  // Compensated correction: L~ and Q^T are also stored as their bf16 rounding
  // errors (Llo, Ctlo) and the output stage adds hi.hi + hi.lo + lo.hi, which
  // removes most of the cancellation error the grouping L~ . Q amplifies.
  bool hilo = false;
  void* Llo = nullptr;   // N x k
  void* Ctlo = nullptr;  // d_out x (B*k)
  // Split T: T = L^T X also as its bf16 rounding errors (Tplo), which the
  // rank-k factor GEMM accumulates as a second B operand, so Q is formed from
  // T to about 16 bits
  bool split_t = false;
  void* Tplo = nullptr;  // (B*k) x d_in
  // Diagnostic: limit of one pipeline wait of the Gram stage in ns (0: the
  // default sm100::kWaitLimitNs). A short limit makes a wait run out, which
  // the stage reports as DYRA_STATUS_WAIT_TIMEOUT before returning.
  unsigned long long gram_wait_ns = 0;
  // Solver of the small systems: 0 the blocked LDL^T factorisation, 1 the
  // Newton-Schulz iteration (at most ns_iters steps; k <= 64)
  int solver = 0;
  int ns_iters = 40;
  // Monarch static part ([DyRA] App. B) in place of Z U^T (r = 0; VPt holds
  // P^T only): Lt holds b2 blocks of b1' x b1 (L_j2 transposed, K-major), Rt
  // b1' blocks of b2' x b2 (R_j1 transposed); Xs is N x d_in and Ms N x b2 b1'
  // of workspace (both also carry the intermediate products).
  const void* Lt = nullptr;
  const void* Rt = nullptr;
  int mb1 = 0, mb2 = 0, mb1o = 0, mb2o = 0;
  void* Xs = nullptr;
  void* Ms = nullptr;
  // ALS updates ([DyRA] Sec. 3.3): 2 is Alg. 1; more run the explicit
  // alternating chain (launch_bf16_als). TG then needs B x k x (d_in + k)
  // floats.
  int half_steps = 2;
};

constexpr int kTraceCtas = 256;  // trace rows per stage (grids are at most this wide)
constexpr int kTraceSlots = 64;  // timestamps per CTA

// Rows per split and split count used for a given T (shared with the
// workspace sizing).
void gram_split(int64_t T, int64_t B, int d_in, int k, int sm_count, int* splits,
                int* split_rows);

int launch_bf16_forward(const Bf16Forward& a, const DeviceInfo& dev, cudaStream_t s);

// Tiling of the projection stage X [V | P] for N rows (k_eff = 0 for the
// weight-only layer): column tile, tile count, CTA pairs or not, and the
// split-K factor chosen when there are too few tiles for the SMs.
struct ProjShape {
  int bn, n_tiles_n, tiles, ksplit, kper, tma_store;
  bool pairs;
};
// pair_min_tiles: pair tiles needed before the projection runs on CTA pairs
// (0: a quarter of the SM count); force_bn: 128, 192 or 256 fixes the column
// tile (0: chosen by the cost model).
ProjShape proj_shape(int64_t N, int d_in, int r, int k_eff, bool use_pairs, int sm_count,
                     int pair_min_tiles = 0, int force_bn = 0);

// ------------------------------------------------------- SIMT (fp32) ----

template <typename T>
struct SimtForward {
  int d_in, d_out, r, k;
  int64_t B, Trows;
  const T* X;
  T* Y;
  const T* VPt;
  const T* U;
  const T* W_res;
  float lambda;
  bool weight_only;
  T* ZL;        // N x (r+k)
  float* TG;    // B x k x (d_in + k)
  T* Tp;        // (B*k) x d_in
  T* Cm;        // (B*k) x d_out
  int* status;
  const T* bias = nullptr;  // d_out values added to Y, or nullptr
  float alpha = 1.f;        // weight of the correction
  // More alternating least-squares updates ([DyRA] Sec. 3.3): half_steps
  // updates in all, L and R alternating, Alg. 1 being the first two. Beyond
  // two, each L update needs the buffers below.
  int half_steps = 2;
  T* Lt = nullptr;       // (B*k) x Trows: the latest L_b, transposed
  T* P2 = nullptr;       // (B*k) x d_in: R_b W_res, the L update's projector before its solve
  float* TG2 = nullptr;  // B x k x (Trows + k): [ (X_b P2_b^T)^T | R_b R_b^T ]
  // Monarch static part ([DyRA] App. B), r = 0: y = x W_hat in the paper's
  // layout, W_hat = P1 L P2^T R with Lblk mb2 blocks of mb1 x mb1o and Rblk
  // mb1o blocks of mb2 x mb2o (row-major, contiguous); Mtmp is N x mb2 mb1o
  const T* Lblk = nullptr;
  const T* Rblk = nullptr;
  int mb1 = 0, mb2 = 0, mb1o = 0, mb2o = 0;
  T* Mtmp = nullptr;
};

template <typename T>
int launch_simt_forward(const SimtForward<T>& a, const DeviceInfo& dev, cudaStream_t s);

// Solve (L^T L + lambda I) T' = T for every instance from the Gram partials
// (the CUDA-core path, and the right updates of further ALS iterations on the
// tensor-core path): every solve block factors G_b itself; alpha scales T'.
template <typename TOut>
int launch_solve(const float* TG, int splits, int64_t B, int k, int d_in, float lambda, TOut* Tp,
                 int* status, cudaStream_t s, bool pdl, unsigned long long* trace = nullptr,
                 float alpha = 1.f);

// Floats per instance of the factor records for correction rank k (0 when
// k > 64: the solve then factors G_b itself).
int factor_record_floats(int k);

// out[row][q * P + p] = in[row][p * Q + q] for `rows` rows of P * Q bf16
// values (P * Q a multiple of 8, at most 49152): the Monarch shuffle.
int launch_grid_transpose(const void* in, void* out, int64_t rows, int P, int Q, int sm_count,
                          cudaStream_t s);

// Newton-Schulz inverse of G_b + lambda I per instance (k <= 64), published
// as factor records behind the instance flags for launch_ltilde's mode 2.
int launch_ns_inverse(const float* G, int64_t B, int k, float lambda, int max_iters, float* MD,
                      int* flags, int* status, cudaStream_t s);

// L~ = L G^-1 per instance, over L (bf16 plans; kernels_simt.cu). mode 0: every
// block factors G_b; 1: the instance's first block factors it and publishes a
// record (MD, flags); 2: every block reads the records another kernel
// published (k <= 64). G: B x k x k fp32 (G_b without the ridge).
// defer_wait (with pdl): the grid launched just before waited for the one
// that wrote G and L before letting this one start; this grid then waits
// for it only before its blocks exit.
// alpha scales the result (the correction weight of the full linear layer);
// Llo (optional, N x k like L) receives the bf16 rounding error of each value.
int launch_ltilde(const float* G, void* L, void* Llo, float* MD, int* flags, int mode, int64_t B,
                  int64_t T, int k, float lambda, float alpha, int* status, cudaStream_t s, bool pdl,
                  bool defer_wait, unsigned long long* trace);
// Dynamic shared memory of one launch_ltilde block, and its rows of L, for this k.
size_t ltilde_smem_bytes(int k);
int ltilde_rows_per_block(int k);

// Pack [V | P]^T: VPt[c][j] = V[j][c] (c < r), P[j][c-r] (c >= r).
template <typename T>
int launch_pack_vp(const T* V, const T* P, T* VPt, int d_in, int r, int k, cudaStream_t s);

}  // namespace dyra
