// dyra_api.cu - the C ABI declared in include/dyra.h.
//
// Owns the plan (shape, device, packed factors, workspace, status word),
// validates every argument before touching the device, and dispatches the
// forward to the tcgen05 kernels (bf16) or the SIMT kernels (fp32).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "dyra.h"
#include "dyra_debug.h"
#include "internal.h"

struct dyra_plan {
  int d_in = 0, d_out = 0, r = 0, k = 0;
  // Monarch static part ([DyRA] App. B) in place of U V^T: n = d_in = d_out =
  // b1 * b2, b2 blocks of b1 x b1 (Lblk) and b1 blocks of b2 x b2 (Rblk); r = 0
  bool monarch = false;
  int mb1 = 0, mb2 = 0, mb1o = 0, mb2o = 0;  // d_in = mb1 mb2, d_out = mb1o mb2o
  void* Lblk = nullptr;
  void* Rblk = nullptr;
  void* Mtmp = nullptr;  // workspace: N x n, the product's intermediate
  size_t cap_Mtmp = 0;
  dyra_dtype_t dtype = DYRA_BF16;
  dyra::DeviceInfo dev;
  bool loaded = false;
  bool force_simt = false;  // DYRA_KERNELS=simt: CUDA-core kernels for bf16 too (debugging)
  bool use_pairs = true;    // DYRA_PAIR=0: single-CTA output stage (comparison)
  int proj_pair_min_tiles = 0;  // DYRA_PROJ_PAIR_MIN=n: projection pairs from n pair tiles
  int proj_bn = 0;              // DYRA_PROJ_BN=128|192|256: projection column tile
  // Where G_b is factored (bf16, k <= 64): by every solve block
  // (DYRA_FACTOR=self), once per instance by the first solve block, which
  // publishes it (DYRA_FACTOR=shared), or by size (unset: every block while
  // the blocks fit the SMs).
  int factor_mode = -1;
  // Compensated correction (low parts of L~ and Q^T, DYRA_HILO=1|0; unset:
  // for single instances of up to 2048 rows, where the output stage is bound
  // by reading U and the extra correction products cost nothing)
  int hilo_mode = -1;
  float lambda = 0.f;
  // full linear layer (dyra_set_linear): Y = static + bias + alpha * correction
  void* bias = nullptr;  // d_out values in the plan dtype (allocated on first use)
  bool has_bias = false;
  float alpha = 1.f;
  // packed factors
  void* VPt = nullptr;   // (r+k) x d_in
  void* U = nullptr;     // d_out x r
  void* W_res = nullptr; // d_out x d_in
  // workspace
  void* Z = nullptr;     // bf16: N x r; fp32: N x (r+k)
  void* L = nullptr;     // bf16: N x k
  float* TG = nullptr;   // bf16: B x k x k (G_b); fp32: B x k x (d_in + k) (T_b, G_b)
  void* Tp = nullptr;    // (B*k) x d_in
  void* Ct = nullptr;    // bf16: d_out x (B*k); fp32: (B*k) x d_out
  void* MD = nullptr;    // bf16, k <= 64: B factor records, then B arrival counters
  void* Llo = nullptr;   // bf16, compensated correction: N x k
  void* Ctlo = nullptr;  // bf16, compensated correction: d_out x (B*k)
  void* Tplo = nullptr;  // bf16, compensated correction: (B*k) x d_in
  size_t cap_Z = 0, cap_L = 0, cap_TG = 0, cap_Tp = 0, cap_Ct = 0, cap_MD = 0;
  // ALS updates per forward (dyra_set_als_steps) and the buffers the further
  // L updates of the CUDA-core kernels use
  int als_half_steps = 2;
  // solver of the small systems (dyra_set_solver)
  int solver = DYRA_SOLVER_LDL;
  int ns_iters = 40;
  void* Lt = nullptr;    // (B*k) x T
  void* P2 = nullptr;    // (B*k) x d_in
  float* TG2 = nullptr;  // B x k x (T + k)
  size_t cap_Lt = 0, cap_P2 = 0, cap_TG2 = 0;
  size_t cap_Llo = 0, cap_Ctlo = 0, cap_Tplo = 0;
  int* status = nullptr;
  size_t factor_bytes = 0;
  cudaEvent_t stage_ev[6] = {};
  bool stage_timing = false;
  bool stage_recorded = false;
  unsigned long long* trace = nullptr;  // timeline buffer (diagnostics)
  unsigned long long gram_wait_ns = 0;  // diagnostic wait limit of the Gram stage (0: default)
  // Captured forwards (CUDA graphs) keyed by their arguments; replayed with
  // one cudaGraphLaunch. Invalidated when workspace or factors change.
  struct GraphEntry {
    const void* X = nullptr;
    void* Y = nullptr;
    int64_t B = 0, T = 0;
    bool weight_only = false;
    cudaGraphExec_t exec = nullptr;
    uint64_t used = 0;
  };
  static constexpr int kGraphSlots = 8;
  GraphEntry graphs[kGraphSlots];
  uint64_t graph_clock = 0;
  cudaStream_t capture_stream = nullptr;
  bool use_graphs = true;
  // dyra_forward_batched_host: two device buffers each for the input and the
  // output chunks, the copy streams and the per-chunk events
  static constexpr int kHostEvents = 16;
  void* hx[2] = {nullptr, nullptr};
  void* hy[2] = {nullptr, nullptr};
  size_t cap_hx[2] = {0, 0}, cap_hy[2] = {0, 0};
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev_start = nullptr;
  cudaEvent_t ev_in[kHostEvents] = {}, ev_comp[kHostEvents] = {}, ev_out[kHostEvents] = {};
};

namespace {

size_t elem_size(dyra_dtype_t t) { return t == DYRA_F32 ? 4 : 2; }

bool fail_alloc_for_test() {
  const char* e = std::getenv("DYRA_TEST_FAIL_ALLOC");
  return e != nullptr && e[0] == '1';
}

int dev_alloc(void** p, size_t bytes) {
  if (fail_alloc_for_test()) return DYRA_ERR_ALLOC;
  if (cudaMalloc(p, bytes) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return DYRA_ERR_ALLOC;
  }
  return DYRA_OK;
}

void dev_free(void*& p) {
  if (p) cudaFree(p);
  p = nullptr;
}

// Grow a workspace buffer to at least `bytes`.
int grow(void*& p, size_t& cap, size_t bytes) {
  if (bytes <= cap) return DYRA_OK;
  dev_free(p);
  cap = 0;
  const size_t rounded = (bytes + 255) & ~static_cast<size_t>(255);
  int rc = dev_alloc(&p, rounded);
  if (rc) return rc;
  cap = rounded;
  return DYRA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void drop_graphs(dyra_plan* p) {
  for (auto& g : p->graphs) {
    if (g.exec) cudaGraphExecDestroy(g.exec);
    g = dyra_plan::GraphEntry();
  }
}

// Run on the plan's device, restoring the caller's device afterwards.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      ok = false;
      return;
    }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

int ensure_workspace_impl(dyra_plan* p, int64_t B, int64_t T);

// Whether a tensor-core forward of B x T rows uses the compensated correction.
bool use_hilo(const dyra_plan* p, int64_t B, int64_t T) {
  if (p->k == 0 || p->dtype != DYRA_BF16 || p->force_simt || p->monarch || p->hilo_mode == 0 ||
      p->als_half_steps != 2)
    return false;
  return p->hilo_mode == 1 || (B == 1 && T <= 2048);
}

// Factor records of the solve plus its per-instance flags (bf16, k <= 64).
size_t factor_bytes(int64_t B, int k) {
  const int rec = dyra::factor_record_floats(k);
  if (rec == 0) return 0;
  return static_cast<size_t>(B) * rec * sizeof(float) + static_cast<size_t>(B) * sizeof(int);
}

// Splits factor_bytes' buffer into its records and counters.
void split_factor_buffer(void* buf, int64_t B, int k, float** md, int** counters) {
  const int rec = dyra::factor_record_floats(k);
  *md = rec ? static_cast<float*>(buf) : nullptr;
  *counters = rec && buf ? reinterpret_cast<int*>(static_cast<float*>(buf) + B * rec) : nullptr;
}

// Grows the workspace; captured graphs point at the old buffers, so any
// growth drops them.
int ensure_workspace(dyra_plan* p, int64_t B, int64_t T) {
  auto caps = [p] {
    return p->cap_Z + p->cap_L + p->cap_TG + p->cap_Tp + p->cap_Ct + p->cap_MD + p->cap_Lt +
           p->cap_P2 + p->cap_TG2 + p->cap_Llo + p->cap_Ctlo + p->cap_Tplo + p->cap_Mtmp;
  };
  const size_t before = caps();
  const void* ptrs[13] = {p->Z,  p->L,  p->TG,  p->Tp,  p->Ct,   p->MD,  p->Lt,
                          p->P2, p->TG2, p->Llo, p->Ctlo, p->Tplo, p->Mtmp};
  const int rc = ensure_workspace_impl(p, B, T);
  const void* now[13] = {p->Z,  p->L,  p->TG,  p->Tp,  p->Ct,   p->MD,  p->Lt,
                         p->P2, p->TG2, p->Llo, p->Ctlo, p->Tplo, p->Mtmp};
  bool moved = before != caps();
  for (int i = 0; i < 13; ++i) moved = moved || ptrs[i] != now[i];
  if (moved) drop_graphs(p);
  return rc;
}

int ensure_workspace_impl(dyra_plan* p, int64_t B, int64_t T) {
  const int64_t N = B * T;
  const size_t es = elem_size(p->dtype);
  const int k = p->k;
  int rc;
  const bool umma = p->dtype == DYRA_BF16 && !p->force_simt;
  const size_t nmid = p->monarch ? static_cast<size_t>(p->mb2) * p->mb1o : 0;
  if (p->monarch) {
    // the intermediate X L-product; on the tensor cores also the shuffled X
    // before it and the shuffled product after it (Z then holds the product)
    void* mt = p->Mtmp;
    const size_t cols = umma ? std::max(static_cast<size_t>(p->d_in), nmid) : nmid;
    if ((rc = grow(mt, p->cap_Mtmp, static_cast<size_t>(N) * cols * es))) return rc;
    p->Mtmp = mt;
  }
  if (umma) {
    const size_t zcols = p->monarch ? nmid : static_cast<size_t>(p->r);
    if ((rc = grow(p->Z, p->cap_Z, static_cast<size_t>(N) * zcols * es))) return rc;
    if (k > 0) {
      if ((rc = grow(p->L, p->cap_L, static_cast<size_t>(N) * k * es))) return rc;
      void* tg = p->TG;
      // more ALS iterations keep L_b^T X_b and L_b^T L_b together in fp32
      const size_t tg_cols = p->als_half_steps > 2 ? static_cast<size_t>(p->d_in) + k : k;
      rc = grow(tg, p->cap_TG, static_cast<size_t>(B) * k * tg_cols * sizeof(float));
      p->TG = static_cast<float*>(tg);
      if (rc) return rc;
      if ((rc = grow(p->Tp, p->cap_Tp, static_cast<size_t>(B) * k * p->d_in * es))) return rc;
      if ((rc = grow(p->Ct, p->cap_Ct, static_cast<size_t>(B) * k * p->d_out * es))) return rc;
      if ((rc = grow(p->MD, p->cap_MD, factor_bytes(B, k)))) return rc;
      if (use_hilo(p, B, T)) {
        if ((rc = grow(p->Llo, p->cap_Llo, static_cast<size_t>(N) * k * es))) return rc;
        if ((rc = grow(p->Ctlo, p->cap_Ctlo, static_cast<size_t>(B) * k * p->d_out * es)))
          return rc;
        if ((rc = grow(p->Tplo, p->cap_Tplo, static_cast<size_t>(B) * k * p->d_in * es)))
          return rc;
      }
    }
  } else {
    if ((rc = grow(p->Z, p->cap_Z, static_cast<size_t>(N) * (p->r + k) * es))) return rc;
    if (k > 0) {
      void* tg = p->TG;
      rc = grow(tg, p->cap_TG, static_cast<size_t>(B) * k * (p->d_in + k) * sizeof(float));
      p->TG = static_cast<float*>(tg);
      if (rc) return rc;
      if ((rc = grow(p->Tp, p->cap_Tp, static_cast<size_t>(B) * k * p->d_in * es))) return rc;
      if ((rc = grow(p->Ct, p->cap_Ct, static_cast<size_t>(B) * k * p->d_out * es))) return rc;
      if (p->als_half_steps > 2) {
        if ((rc = grow(p->Lt, p->cap_Lt, static_cast<size_t>(B) * k * T * es))) return rc;
        if ((rc = grow(p->P2, p->cap_P2, static_cast<size_t>(B) * k * p->d_in * es))) return rc;
        void* tg2 = p->TG2;
        rc = grow(tg2, p->cap_TG2, static_cast<size_t>(B) * k * (T + k) * sizeof(float));
        p->TG2 = static_cast<float*>(tg2);
        if (rc) return rc;
      }
    }
  }
  return DYRA_OK;
}

// Launch a forward through a cached CUDA graph when possible: one
// cudaGraphLaunch replaces its kernel launches (five for the tensor-core
// path, seven for the CUDA-core path) and, for the tensor-core path, twelve
// tensor-map encodings. Graphs are not used while the caller's stream is being
// captured (the launches then go into the caller's graph), when `direct` is
// set (stage timing or tracing), or when DYRA_GRAPHS=0. `launch(stream)`
// enqueues the forward's kernels on `stream` and returns 0 on success.
template <class Launch>
int launch_maybe_graph(dyra_plan* p, const void* X, void* Y, int64_t B, int64_t T,
                       bool weight_only, bool direct, cudaStream_t s, const Launch& launch) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (!p->use_graphs || direct || cudaStreamIsCapturing(s, &cs) != cudaSuccess ||
      cs != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return launch(s);
  }
  dyra_plan::GraphEntry* hit = nullptr;
  for (auto& g : p->graphs)
    if (g.exec && g.X == X && g.Y == Y && g.B == B && g.T == T && g.weight_only == weight_only)
      hit = &g;
  if (!hit) {
    if (!p->capture_stream &&
        cudaStreamCreateWithFlags(&p->capture_stream, cudaStreamNonBlocking) != cudaSuccess)
      return launch(s);
    cudaGraph_t graph = nullptr;
    if (cudaStreamBeginCapture(p->capture_stream, cudaStreamCaptureModeThreadLocal) !=
        cudaSuccess) {
      cudaGetLastError();
      return launch(s);
    }
    const int lrc = launch(p->capture_stream);
    const cudaError_t ec = cudaStreamEndCapture(p->capture_stream, &graph);
    cudaGraphExec_t exec = nullptr;
    if (lrc != 0 || ec != cudaSuccess || graph == nullptr ||
        cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      cudaGetLastError();
      return launch(s);
    }
    cudaGraphDestroy(graph);
    hit = &p->graphs[0];
    for (auto& g : p->graphs) {
      if (!g.exec) {
        hit = &g;
        break;
      }
      if (g.used < hit->used) hit = &g;
    }
    if (hit->exec) cudaGraphExecDestroy(hit->exec);
    hit->X = X;
    hit->Y = Y;
    hit->B = B;
    hit->T = T;
    hit->weight_only = weight_only;
    hit->exec = exec;
  }
  hit->used = ++p->graph_clock;
  return cudaGraphLaunch(hit->exec, s) == cudaSuccess ? 0 : -1;
}

int run_forward(dyra_plan* p, const void* X, void* Y, int64_t B, int64_t T, bool weight_only,
                cudaStream_t s) {
  if (p == nullptr) return DYRA_ERR_INVALID_ARG;
  if (B < 0 || T < 0) return DYRA_ERR_INVALID_ARG;
  const int64_t N = B * T;
  if (N == 0) return DYRA_OK;
  if (X == nullptr || Y == nullptr) return DYRA_ERR_INVALID_ARG;
  if (N > (static_cast<int64_t>(1) << 31) - 1 || B * static_cast<int64_t>(p->k) > (1 << 30))
    return DYRA_ERR_INVALID_ARG;
  if (!p->loaded) return DYRA_ERR_NOT_LOADED;
  if (!aligned16(X) || !aligned16(Y)) return DYRA_ERR_ALIGNMENT;
  const bool correct = !weight_only && p->k > 0;
  if (correct && p->lambda == 0.f && T < p->k) return DYRA_ERR_RANK_DEFICIENT;

  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  int rc = ensure_workspace(p, B, T);
  if (rc) return rc;

  if (p->dtype == DYRA_BF16 && !p->force_simt) {
    dyra::Bf16Forward a;
    a.d_in = p->d_in;
    a.d_out = p->d_out;
    a.r = p->r;
    a.k = p->k;
    a.B = B;
    a.T = T;
    a.X = X;
    a.Y = Y;
    a.VPt = p->VPt;
    a.U = p->U;
    a.W_res = p->W_res;
    a.lambda = p->lambda;
    a.weight_only = !correct;
    a.Z = p->Z;
    a.L = p->L;
    a.TG = p->TG;
    a.Tp = p->Tp;
    a.Ct = p->Ct;
    split_factor_buffer(correct ? p->MD : nullptr, B, p->k, &a.MD, &a.counters);
    a.factor_mode = p->factor_mode;
    a.splits = 1;
    a.split_rows = 64;
    if (correct) dyra::gram_split(T, B, p->d_in, p->k, p->dev.sm_count, &a.splits, &a.split_rows);
    a.status = p->status;
    a.stage_events = p->stage_timing ? p->stage_ev : nullptr;
    a.trace = p->trace;
    a.gram_wait_ns = p->gram_wait_ns;
    a.half_steps = p->als_half_steps;
    a.solver = p->solver;
    a.ns_iters = p->ns_iters;
    a.use_pairs = p->use_pairs;
    a.proj_pair_min_tiles = p->proj_pair_min_tiles;
    a.proj_bn = p->proj_bn;
    a.bias = p->has_bias ? p->bias : nullptr;
    a.alpha = p->alpha;
    a.hilo = correct && use_hilo(p, B, T);
    a.Llo = a.hilo ? p->Llo : nullptr;
    a.Ctlo = a.hilo ? p->Ctlo : nullptr;
    a.split_t = a.hilo;
    a.Tplo = a.hilo ? p->Tplo : nullptr;
    if (p->monarch) {
      a.Lt = p->Lblk;
      a.Rt = p->Rblk;
      a.mb1 = p->mb1;
      a.mb2 = p->mb2;
      a.mb1o = p->mb1o;
      a.mb2o = p->mb2o;
      a.Xs = p->Mtmp;
      a.Ms = p->Z;
    }
    rc = launch_maybe_graph(p, X, Y, B, T, a.weight_only, a.stage_events || a.trace, s,
                            [&](cudaStream_t st) { return dyra::launch_bf16_forward(a, p->dev, st); });
    p->stage_recorded = p->stage_timing && rc == 0;
  } else if (p->dtype == DYRA_BF16) {
    dyra::SimtForward<__nv_bfloat16> a;
    a.d_in = p->d_in;
    a.d_out = p->d_out;
    a.r = p->r;
    a.k = p->k;
    a.B = B;
    a.Trows = T;
    a.X = static_cast<const __nv_bfloat16*>(X);
    a.Y = static_cast<__nv_bfloat16*>(Y);
    a.VPt = static_cast<const __nv_bfloat16*>(p->VPt);
    a.U = static_cast<const __nv_bfloat16*>(p->U);
    a.W_res = static_cast<const __nv_bfloat16*>(p->W_res);
    a.lambda = p->lambda;
    a.weight_only = !correct;
    a.ZL = static_cast<__nv_bfloat16*>(p->Z);
    a.TG = p->TG;
    a.Tp = static_cast<__nv_bfloat16*>(p->Tp);
    a.Cm = static_cast<__nv_bfloat16*>(p->Ct);
    a.status = p->status;
    a.bias = p->has_bias ? static_cast<const __nv_bfloat16*>(p->bias) : nullptr;
    a.alpha = p->alpha;
    a.half_steps = p->als_half_steps;
    a.Lt = static_cast<__nv_bfloat16*>(p->Lt);
    a.P2 = static_cast<__nv_bfloat16*>(p->P2);
    a.TG2 = p->TG2;
    if (p->monarch) {
      a.Lblk = static_cast<const __nv_bfloat16*>(p->Lblk);
      a.Rblk = static_cast<const __nv_bfloat16*>(p->Rblk);
      a.mb1 = p->mb1;
      a.mb2 = p->mb2;
      a.mb1o = p->mb1o;
      a.mb2o = p->mb2o;
      a.Mtmp = static_cast<__nv_bfloat16*>(p->Mtmp);
    }
    rc = launch_maybe_graph(p, X, Y, B, T, a.weight_only, false, s,
                            [&](cudaStream_t st) { return dyra::launch_simt_forward(a, p->dev, st); });
  } else {
    dyra::SimtForward<float> a;
    a.d_in = p->d_in;
    a.d_out = p->d_out;
    a.r = p->r;
    a.k = p->k;
    a.B = B;
    a.Trows = T;
    a.X = static_cast<const float*>(X);
    a.Y = static_cast<float*>(Y);
    a.VPt = static_cast<const float*>(p->VPt);
    a.U = static_cast<const float*>(p->U);
    a.W_res = static_cast<const float*>(p->W_res);
    a.lambda = p->lambda;
    a.weight_only = !correct;
    a.ZL = static_cast<float*>(p->Z);
    a.TG = p->TG;
    a.Tp = static_cast<float*>(p->Tp);
    a.Cm = static_cast<float*>(p->Ct);
    a.status = p->status;
    a.bias = p->has_bias ? static_cast<const float*>(p->bias) : nullptr;
    a.alpha = p->alpha;
    a.half_steps = p->als_half_steps;
    a.Lt = static_cast<float*>(p->Lt);
    a.P2 = static_cast<float*>(p->P2);
    a.TG2 = p->TG2;
    if (p->monarch) {
      a.Lblk = static_cast<const float*>(p->Lblk);
      a.Rblk = static_cast<const float*>(p->Rblk);
      a.mb1 = p->mb1;
      a.mb2 = p->mb2;
      a.mb1o = p->mb1o;
      a.mb2o = p->mb2o;
      a.Mtmp = static_cast<float*>(p->Mtmp);
    }
    rc = launch_maybe_graph(p, X, Y, B, T, a.weight_only, false, s,
                            [&](cudaStream_t st) { return dyra::launch_simt_forward(a, p->dev, st); });
  }
  if (rc != 0) {
    cudaGetLastError();
    return DYRA_ERR_CUDA;
  }
  return DYRA_OK;
}

}  // namespace

namespace dyra {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (swizzle_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  if (swizzle_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  if (swizzle_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  cuuint64_t d[5];
  cuuint64_t st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  std::memset(map, 0, sizeof(*map));
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
            const_cast<void*>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dyra

extern "C" {

const char* dyra_error_string(int code) {
  switch (code) {
    case DYRA_OK: return "ok";
    case DYRA_ERR_INVALID_ARG: return "invalid argument";
    case DYRA_ERR_NOT_LOADED: return "factors not loaded";
    case DYRA_ERR_ALIGNMENT: return "misaligned pointer or size";
    case DYRA_ERR_RANK_DEFICIENT: return "lambda == 0 and fewer rows than the correction rank";
    case DYRA_ERR_ALLOC: return "device allocation failed";
    case DYRA_ERR_CUDA: return "CUDA call failed";
    case DYRA_ERR_UNSUPPORTED: return "device is not compute capability 10.0";
    case DYRA_ERR_DEVICE: return "device status raised";
    default: return "unknown error";
  }
}

static int plan_create_impl(dyra_plan_t* out, int d_in, int d_out, int r, int k,
                            dyra_dtype_t dtype);

int dyra_plan_create(dyra_plan_t* out, int d_in, int d_out, int r, int k, dyra_dtype_t dtype) {
  if (out == nullptr) return DYRA_ERR_INVALID_ARG;
  if (dtype != DYRA_F32 && dtype != DYRA_BF16) return DYRA_ERR_INVALID_ARG;
  if (d_in < 1 || d_out < 1 || r < 1 || k < 0 || k > 128) return DYRA_ERR_INVALID_ARG;
  const int m = d_in < d_out ? d_in : d_out;
  if (r + k > m) return DYRA_ERR_INVALID_ARG;
  if (dtype == DYRA_BF16 && (d_in % 8 || d_out % 8 || r % 8 || k % 8)) return DYRA_ERR_ALIGNMENT;
  return plan_create_impl(out, d_in, d_out, r, k, dtype);
}

int dyra_plan_create_monarch_rect(dyra_plan_t* out, int b1, int b2, int b1o, int b2o, int k,
                                  dyra_dtype_t dtype) {
  if (out == nullptr) return DYRA_ERR_INVALID_ARG;
  if (dtype != DYRA_F32 && dtype != DYRA_BF16) return DYRA_ERR_INVALID_ARG;
  if (b1 < 1 || b2 < 1 || b1o < 1 || b2o < 1 || k < 0 || k > 128) return DYRA_ERR_INVALID_ARG;
  const int64_t d_in = static_cast<int64_t>(b1) * b2, d_out = static_cast<int64_t>(b1o) * b2o;
  const int64_t nmid = static_cast<int64_t>(b2) * b1o;
  if (d_in > 49152 || d_out > 49152 || nmid > 49152 || k > std::min(d_in, d_out))
    return DYRA_ERR_INVALID_ARG;
  // bf16: 16-byte rows, and (tensor cores) 16-byte block offsets within rows
  if (dtype == DYRA_BF16 && (d_in % 8 || d_out % 8 || k % 8 || b1 % 8 || b2 % 8))
    return DYRA_ERR_ALIGNMENT;
  const int rc = plan_create_impl(out, static_cast<int>(d_in), static_cast<int>(d_out), 0, k,
                                  dtype);
  if (rc == DYRA_OK) {
    (*out)->monarch = true;
    (*out)->mb1 = b1;
    (*out)->mb2 = b2;
    (*out)->mb1o = b1o;
    (*out)->mb2o = b2o;
  }
  return rc;
}

int dyra_plan_create_monarch(dyra_plan_t* out, int n, int b1, int b2, int k, dyra_dtype_t dtype) {
  if (out == nullptr || b1 < 1 || b2 < 1 || n != b1 * b2) return DYRA_ERR_INVALID_ARG;
  return dyra_plan_create_monarch_rect(out, b1, b2, b1, b2, k, dtype);
}

static int plan_create_impl(dyra_plan_t* out, int d_in, int d_out, int r, int k,
                            dyra_dtype_t dtype) {

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return DYRA_ERR_CUDA;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return DYRA_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return DYRA_ERR_UNSUPPORTED;

  dyra_plan* p = new (std::nothrow) dyra_plan();
  if (!p) return DYRA_ERR_ALLOC;
  p->d_in = d_in;
  p->d_out = d_out;
  p->r = r;
  p->k = k;
  p->dtype = dtype;
  p->dev.device = dev;
  p->dev.sm_count = prop.multiProcessorCount;
  p->dev.max_smem_optin = static_cast<int>(prop.sharedMemPerBlockOptin);
  p->dev.smem_per_sm = static_cast<int>(prop.sharedMemPerMultiprocessor);
  p->dev.smem_reserved = static_cast<int>(prop.reservedSharedMemPerBlock);
  p->dev.cc_major = prop.major;
  p->dev.cc_minor = prop.minor;
  const char* kv = std::getenv("DYRA_KERNELS");
  p->force_simt = kv != nullptr && std::strcmp(kv, "simt") == 0;
  const char* pv = std::getenv("DYRA_PAIR");
  p->use_pairs = !(pv != nullptr && pv[0] == '0');
  const char* ppv = std::getenv("DYRA_PROJ_PAIR_MIN");
  p->proj_pair_min_tiles = ppv ? std::atoi(ppv) : 0;
  const char* pbv = std::getenv("DYRA_PROJ_BN");
  p->proj_bn = pbv ? std::atoi(pbv) : 0;
  if (p->proj_bn != 128 && p->proj_bn != 192 && p->proj_bn != 256) p->proj_bn = 0;
  const char* fv = std::getenv("DYRA_FACTOR");
  p->factor_mode = fv == nullptr                     ? -1
                   : std::strcmp(fv, "self") == 0   ? 0
                   : std::strcmp(fv, "shared") == 0 ? 1
                                                    : -1;
  const char* hv = std::getenv("DYRA_HILO");
  p->hilo_mode = hv == nullptr ? -1 : (hv[0] == '1' ? 1 : (hv[0] == '0' ? 0 : -1));
  const char* gv = std::getenv("DYRA_GRAPHS");
  p->use_graphs = !(gv != nullptr && gv[0] == '0');
  void* st = nullptr;
  if (dev_alloc(&st, 256) != DYRA_OK) {
    delete p;
    return DYRA_ERR_ALLOC;
  }
  p->status = static_cast<int*>(st);
  if (cudaMemset(p->status, 0, sizeof(int)) != cudaSuccess) {
    dev_free(st);
    delete p;
    return DYRA_ERR_CUDA;
  }
  *out = p;
  return DYRA_OK;
}

int dyra_load_factors(dyra_plan_t p, const void* U, const void* V, const void* P,
                      const void* W_res, float lambda, dyra_stream_t stream) {
  if (p == nullptr || U == nullptr || V == nullptr || p->monarch) return DYRA_ERR_INVALID_ARG;
  if (p->k > 0 && (P == nullptr || W_res == nullptr)) return DYRA_ERR_INVALID_ARG;
  if (!(lambda >= 0.f) || !std::isfinite(lambda)) return DYRA_ERR_INVALID_ARG;
  if (!aligned16(U) || !aligned16(V) || (p->k > 0 && (!aligned16(P) || !aligned16(W_res))))
    return DYRA_ERR_ALIGNMENT;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = elem_size(p->dtype);
  const size_t vpt = static_cast<size_t>(p->r + p->k) * p->d_in * es;
  const size_t ub = static_cast<size_t>(p->d_out) * p->r * es;
  const size_t wb = p->k > 0 ? static_cast<size_t>(p->d_out) * p->d_in * es : 0;
  int rc;
  if (!p->VPt && (rc = dev_alloc(&p->VPt, vpt))) return rc;
  if (!p->U && (rc = dev_alloc(&p->U, ub))) return rc;
  if (wb && !p->W_res && (rc = dev_alloc(&p->W_res, wb))) return rc;
  p->factor_bytes = vpt + ub + wb;
  if (cudaMemcpyAsync(p->U, U, ub, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DYRA_ERR_CUDA;
  if (wb && cudaMemcpyAsync(p->W_res, W_res, wb, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DYRA_ERR_CUDA;
  if (p->dtype == DYRA_BF16)
    rc = dyra::launch_pack_vp(static_cast<const __nv_bfloat16*>(V),
                              static_cast<const __nv_bfloat16*>(P),
                              static_cast<__nv_bfloat16*>(p->VPt), p->d_in, p->r, p->k, s);
  else
    rc = dyra::launch_pack_vp(static_cast<const float*>(V), static_cast<const float*>(P),
                              static_cast<float*>(p->VPt), p->d_in, p->r, p->k, s);
  if (rc) return DYRA_ERR_CUDA;
  p->lambda = lambda;
  p->loaded = true;
  drop_graphs(p);  // lambda is baked into captured launches
  return DYRA_OK;
}

int dyra_set_linear(dyra_plan_t p, const void* bias, float alpha, dyra_stream_t stream) {
  if (p == nullptr || !std::isfinite(alpha)) return DYRA_ERR_INVALID_ARG;
  if (bias != nullptr && !aligned16(bias)) return DYRA_ERR_ALIGNMENT;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  const size_t bytes = static_cast<size_t>(p->d_out) * elem_size(p->dtype);
  int rc;
  if (bias != nullptr) {
    if (!p->bias && (rc = dev_alloc(&p->bias, bytes))) return rc;
    if (cudaMemcpyAsync(p->bias, bias, bytes, cudaMemcpyDeviceToDevice,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
      cudaGetLastError();
      return DYRA_ERR_CUDA;
    }
  }
  p->has_bias = bias != nullptr;
  p->alpha = alpha;
  drop_graphs(p);  // the bias pointer and alpha are baked into captured launches
  return DYRA_OK;
}

int dyra_set_solver(dyra_plan_t p, int solver, int max_iters) {
  if (p == nullptr || (solver != DYRA_SOLVER_LDL && solver != DYRA_SOLVER_NEWTON_SCHULZ) ||
      max_iters < 1 || max_iters > 200)
    return DYRA_ERR_INVALID_ARG;
  const bool umma = p->dtype == DYRA_BF16 && !p->force_simt;
  if (solver == DYRA_SOLVER_NEWTON_SCHULZ && (!umma || p->k == 0 || p->k > 64))
    return DYRA_ERR_UNSUPPORTED;
  p->solver = solver;
  p->ns_iters = max_iters;
  drop_graphs(p);  // captured forwards hold the old solver
  return DYRA_OK;
}

int dyra_set_als_steps(dyra_plan_t p, int half_steps) {
  if (p == nullptr || half_steps < 2 || half_steps > 64) return DYRA_ERR_INVALID_ARG;
  // the Monarch static part runs one ALS step on the tensor cores
  if (p->monarch && p->dtype == DYRA_BF16 && !p->force_simt && half_steps != 2)
    return DYRA_ERR_UNSUPPORTED;
  p->als_half_steps = half_steps;
  drop_graphs(p);  // captured forwards hold the old count
  return DYRA_OK;
}

int dyra_forward_batched_host(dyra_plan_t p, const void* X, void* Y, int64_t B, int64_t T,
                              dyra_stream_t stream) {
  if (p == nullptr || B < 0 || T < 0) return DYRA_ERR_INVALID_ARG;
  if (B * T == 0) return DYRA_OK;
  if (X == nullptr || Y == nullptr) return DYRA_ERR_INVALID_ARG;
  if (!p->loaded) return DYRA_ERR_NOT_LOADED;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = elem_size(p->dtype);
  // Chunks of whole instances (each instance's correction needs all of its
  // rows): up to kHostEvents of them, at least about 1 MiB of input each.
  const size_t inst_in = static_cast<size_t>(T) * p->d_in * es;
  const size_t inst_out = static_cast<size_t>(T) * p->d_out * es;
  int64_t per = std::max<int64_t>(1, (B + dyra_plan::kHostEvents - 1) / dyra_plan::kHostEvents);
  per = std::max<int64_t>(per, std::min<int64_t>(B, static_cast<int64_t>((1u << 20) / inst_in) + 1));
  const int64_t chunks = (B + per - 1) / per;
  int rc;
  for (int i = 0; i < 2; ++i) {
    if ((rc = grow(p->hx[i], p->cap_hx[i], per * inst_in))) return rc;
    if ((rc = grow(p->hy[i], p->cap_hy[i], per * inst_out))) return rc;
  }
  auto make_stream = [](cudaStream_t* st) {
    return *st || cudaStreamCreateWithFlags(st, cudaStreamNonBlocking) == cudaSuccess;
  };
  auto make_event = [](cudaEvent_t* e) {
    return *e || cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  };
  bool ok = make_stream(&p->h2d) && make_stream(&p->d2h) && make_event(&p->ev_start);
  for (int i = 0; ok && i < dyra_plan::kHostEvents; ++i)
    ok = make_event(&p->ev_in[i]) && make_event(&p->ev_comp[i]) && make_event(&p->ev_out[i]);
  if (!ok) {
    cudaGetLastError();
    return DYRA_ERR_CUDA;
  }
  // chunk c: X -> hx[c % 2] on h2d, the forward on `stream`, hy[c % 2] -> Y on d2h.
  // hx[c % 2] is rewritten once the forward of chunk c - 2 has read it, hy[c % 2]
  // once the copy of chunk c - 2 has read it; `stream` then waits for the last copy.
  const char* xs = static_cast<const char*>(X);
  char* ys = static_cast<char*>(Y);
  bool err = cudaEventRecord(p->ev_start, s) != cudaSuccess ||
             cudaStreamWaitEvent(p->h2d, p->ev_start, 0) != cudaSuccess;
  for (int64_t c = 0; !err && c < chunks; ++c) {
    const int64_t b0 = c * per, bc = std::min<int64_t>(per, B - b0);
    const int buf = static_cast<int>(c % 2);
    const int e = static_cast<int>(c % dyra_plan::kHostEvents);
    const int e2 = static_cast<int>((c + dyra_plan::kHostEvents - 2) % dyra_plan::kHostEvents);
    if (c >= 2) err = cudaStreamWaitEvent(p->h2d, p->ev_comp[e2], 0) != cudaSuccess;
    err = err || cudaMemcpyAsync(p->hx[buf], xs + b0 * inst_in, bc * inst_in,
                                 cudaMemcpyHostToDevice, p->h2d) != cudaSuccess;
    err = err || cudaEventRecord(p->ev_in[e], p->h2d) != cudaSuccess;
    err = err || cudaStreamWaitEvent(s, p->ev_in[e], 0) != cudaSuccess;
    if (c >= 2) err = err || cudaStreamWaitEvent(s, p->ev_out[e2], 0) != cudaSuccess;
    if (err) break;
    rc = run_forward(p, p->hx[buf], p->hy[buf], bc, T, false, s);
    if (rc) return rc;
    err = cudaEventRecord(p->ev_comp[e], s) != cudaSuccess ||
          cudaStreamWaitEvent(p->d2h, p->ev_comp[e], 0) != cudaSuccess ||
          cudaMemcpyAsync(ys + b0 * inst_out, p->hy[buf], bc * inst_out, cudaMemcpyDeviceToHost,
                          p->d2h) != cudaSuccess ||
          cudaEventRecord(p->ev_out[e], p->d2h) != cudaSuccess;
    if (!err && c == chunks - 1) err = cudaStreamWaitEvent(s, p->ev_out[e], 0) != cudaSuccess;
  }
  if (err) {
    cudaGetLastError();
    return DYRA_ERR_CUDA;
  }
  return DYRA_OK;
}

int dyra_load_monarch(dyra_plan_t p, const void* Lblocks, const void* Rblocks, const void* P,
                      const void* W_res, float lambda, dyra_stream_t stream) {
  if (p == nullptr || !p->monarch || Lblocks == nullptr || Rblocks == nullptr)
    return DYRA_ERR_INVALID_ARG;
  if (p->k > 0 && (P == nullptr || W_res == nullptr)) return DYRA_ERR_INVALID_ARG;
  if (!(lambda >= 0.f) || !std::isfinite(lambda)) return DYRA_ERR_INVALID_ARG;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = elem_size(p->dtype);
  const size_t n = static_cast<size_t>(p->d_in);
  const size_t lb = static_cast<size_t>(p->mb2) * p->mb1 * p->mb1o * es;
  const size_t rb = static_cast<size_t>(p->mb1o) * p->mb2 * p->mb2o * es;
  const size_t vpt = static_cast<size_t>(p->k) * n * es;
  const size_t wb = p->k > 0 ? n * static_cast<size_t>(p->d_out) * es : 0;
  const bool umma = p->dtype == DYRA_BF16 && !p->force_simt;
  int rc;
  if (!p->Lblk && (rc = dev_alloc(&p->Lblk, lb))) return rc;
  if (!p->Rblk && (rc = dev_alloc(&p->Rblk, rb))) return rc;
  if (vpt && !p->VPt && (rc = dev_alloc(&p->VPt, vpt))) return rc;
  if (wb && !p->W_res && (rc = dev_alloc(&p->W_res, wb))) return rc;
  p->factor_bytes = lb + rb + vpt + wb;
  if (umma) {
    // the tensor cores take each block transposed (K-major): L_j2^T and R_j1^T
    if (dyra::launch_grid_transpose(Lblocks, p->Lblk, p->mb2, p->mb1, p->mb1o, p->dev.sm_count,
                                    s) ||
        dyra::launch_grid_transpose(Rblocks, p->Rblk, p->mb1o, p->mb2, p->mb2o, p->dev.sm_count,
                                    s))
      return DYRA_ERR_CUDA;
  } else if (cudaMemcpyAsync(p->Lblk, Lblocks, lb, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
             cudaMemcpyAsync(p->Rblk, Rblocks, rb, cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
    return DYRA_ERR_CUDA;
  }
  if (wb && cudaMemcpyAsync(p->W_res, W_res, wb, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DYRA_ERR_CUDA;
  if (vpt) {  // P^T (k x n): the projection's B operand, as [V | P]^T with r = 0
    if (p->dtype == DYRA_BF16)
      rc = dyra::launch_pack_vp(static_cast<const __nv_bfloat16*>(P),
                                static_cast<const __nv_bfloat16*>(P),
                                static_cast<__nv_bfloat16*>(p->VPt), p->d_in, 0, p->k, s);
    else
      rc = dyra::launch_pack_vp(static_cast<const float*>(P), static_cast<const float*>(P),
                                static_cast<float*>(p->VPt), p->d_in, 0, p->k, s);
    if (rc) return DYRA_ERR_CUDA;
  }
  p->lambda = lambda;
  p->loaded = true;
  drop_graphs(p);
  return DYRA_OK;
}

int dyra_forward(dyra_plan_t p, const void* X, void* Y, int64_t N, dyra_stream_t stream) {
  return run_forward(p, X, Y, 1, N, false, reinterpret_cast<cudaStream_t>(stream));
}

int dyra_forward_batched(dyra_plan_t p, const void* X, void* Y, int64_t B, int64_t T,
                         dyra_stream_t stream) {
  return run_forward(p, X, Y, B, T, false, reinterpret_cast<cudaStream_t>(stream));
}

int dyra_forward_weight_only(dyra_plan_t p, const void* X, void* Y, int64_t N,
                             dyra_stream_t stream) {
  return run_forward(p, X, Y, 1, N, true, reinterpret_cast<cudaStream_t>(stream));
}

int dyra_reserve(dyra_plan_t p, int64_t B, int64_t T) {
  if (p == nullptr || B < 0 || T < 0) return DYRA_ERR_INVALID_ARG;
  if (B * T == 0) return DYRA_OK;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  return ensure_workspace(p, B, T);
}

int dyra_last_status(dyra_plan_t p) {
  if (p == nullptr) return DYRA_ERR_INVALID_ARG;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return DYRA_ERR_CUDA;
  int st = 0;
  if (cudaMemcpy(&st, p->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DYRA_ERR_CUDA;
  if (cudaMemset(p->status, 0, sizeof(int)) != cudaSuccess) return DYRA_ERR_CUDA;
  return st;
}

int dyra_plan_destroy(dyra_plan_t p) {
  if (p == nullptr) return DYRA_OK;
  {
    DeviceGuard g(p->dev.device);
    cudaDeviceSynchronize();
    dev_free(p->VPt);
    dev_free(p->U);
    dev_free(p->W_res);
    dev_free(p->bias);
    dev_free(p->Lblk);
    dev_free(p->Rblk);
    dev_free(p->Mtmp);
    dev_free(p->Z);
    dev_free(p->L);
    void* tg = p->TG;
    dev_free(tg);
    dev_free(p->Tp);
    dev_free(p->Ct);
    dev_free(p->MD);
    dev_free(p->Lt);
    dev_free(p->P2);
    void* tg2 = p->TG2;
    dev_free(tg2);
    dev_free(p->Llo);
    dev_free(p->Ctlo);
    dev_free(p->Tplo);
    void* st = p->status;
    dev_free(st);
    for (auto& e : p->stage_ev)
      if (e) cudaEventDestroy(e);
    if (p->trace) cudaFree(p->trace);
    drop_graphs(p);
    if (p->capture_stream) cudaStreamDestroy(p->capture_stream);
    for (int i = 0; i < 2; ++i) {
      dev_free(p->hx[i]);
      dev_free(p->hy[i]);
    }
    if (p->h2d) cudaStreamDestroy(p->h2d);
    if (p->d2h) cudaStreamDestroy(p->d2h);
    if (p->ev_start) cudaEventDestroy(p->ev_start);
    for (int i = 0; i < dyra_plan::kHostEvents; ++i) {
      if (p->ev_in[i]) cudaEventDestroy(p->ev_in[i]);
      if (p->ev_comp[i]) cudaEventDestroy(p->ev_comp[i]);
      if (p->ev_out[i]) cudaEventDestroy(p->ev_out[i]);
    }
  }
  delete p;
  return DYRA_OK;
}

int dyra_debug_buffer(dyra_plan_t p, int which, const void** ptr, size_t* bytes) {
  if (p == nullptr || ptr == nullptr || bytes == nullptr) return DYRA_ERR_INVALID_ARG;
  switch (which) {
    case DYRA_BUF_Z: *ptr = p->Z; *bytes = p->cap_Z; break;
    case DYRA_BUF_L: *ptr = p->L; *bytes = p->cap_L; break;
    case DYRA_BUF_TG: *ptr = p->TG; *bytes = p->cap_TG; break;
    case DYRA_BUF_TP: *ptr = p->Tp; *bytes = p->cap_Tp; break;
    case DYRA_BUF_CT: *ptr = p->Ct; *bytes = p->cap_Ct; break;
    default: return DYRA_ERR_INVALID_ARG;
  }
  return DYRA_OK;
}

int dyra_debug_copy(dyra_plan_t p, int which, void* dst, size_t bytes) {
  const void* src = nullptr;
  size_t cap = 0;
  int rc = dyra_debug_buffer(p, which, &src, &cap);
  if (rc) return rc;
  if (dst == nullptr || src == nullptr || bytes > cap) return DYRA_ERR_INVALID_ARG;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return DYRA_ERR_CUDA;
  return cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost) == cudaSuccess ? DYRA_OK
                                                                            : DYRA_ERR_CUDA;
}

int dyra_debug_set_stage_timing(dyra_plan_t p, int enable) {
  if (p == nullptr) return DYRA_ERR_INVALID_ARG;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  if (enable && !p->stage_ev[0]) {
    for (auto& e : p->stage_ev)
      if (cudaEventCreate(&e) != cudaSuccess) return DYRA_ERR_CUDA;
  }
  p->stage_timing = enable != 0 && p->dtype == DYRA_BF16 && !p->force_simt && !p->monarch;
  p->stage_recorded = false;
  return p->stage_timing || !enable ? DYRA_OK : DYRA_ERR_INVALID_ARG;
}

int dyra_debug_set_wait_limit(dyra_plan_t p, int stage, uint64_t ns) {
  if (p == nullptr) return DYRA_ERR_INVALID_ARG;
  if (stage != 1) return DYRA_ERR_UNSUPPORTED;
  p->gram_wait_ns = ns;
  drop_graphs(p);  // the limit is a launch parameter of captured forwards
  return DYRA_OK;
}

int dyra_debug_stage_times(dyra_plan_t p, float* ms5) {
  if (p == nullptr || ms5 == nullptr || !p->stage_recorded) return DYRA_ERR_INVALID_ARG;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  if (cudaEventSynchronize(p->stage_ev[5]) != cudaSuccess) return DYRA_ERR_CUDA;
  // The events bracket the launches in stream order: proj, gram, rfactor,
  // solve, out; the result is in stage order (proj, gram, solve, rfactor, out).
  static const int kSlot[5] = {0, 1, 3, 2, 4};
  for (int i = 0; i < 5; ++i) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p->stage_ev[i], p->stage_ev[i + 1]) != cudaSuccess)
      return DYRA_ERR_CUDA;
    ms5[kSlot[i]] = ms;
  }
  return DYRA_OK;
}

int dyra_debug_set_trace(dyra_plan_t p, int enable) {
  if (p == nullptr) return DYRA_ERR_INVALID_ARG;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  if (!enable) {
    if (p->trace) cudaFree(p->trace);
    p->trace = nullptr;
    return DYRA_OK;
  }
  const size_t bytes = dyra_debug_trace_bytes();
  if (!p->trace) {
    void* t = nullptr;
    int rc = dev_alloc(&t, bytes);
    if (rc) return rc;
    p->trace = static_cast<unsigned long long*>(t);
  }
  return cudaMemset(p->trace, 0, bytes) == cudaSuccess ? DYRA_OK : DYRA_ERR_CUDA;
}

size_t dyra_debug_trace_bytes(void) {
  return static_cast<size_t>(5) * dyra::kTraceCtas * dyra::kTraceSlots * sizeof(unsigned long long);
}

int dyra_debug_trace_copy(dyra_plan_t p, void* dst, size_t bytes) {
  if (p == nullptr || dst == nullptr || p->trace == nullptr || bytes > dyra_debug_trace_bytes())
    return DYRA_ERR_INVALID_ARG;
  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return DYRA_ERR_CUDA;
  return cudaMemcpy(dst, p->trace, bytes, cudaMemcpyDeviceToHost) == cudaSuccess ? DYRA_OK
                                                                                  : DYRA_ERR_CUDA;
}

int dyra_debug_gram_split(dyra_plan_t p, int64_t B, int64_t T, int* splits, int* split_rows) {
  if (p == nullptr || splits == nullptr || split_rows == nullptr || B < 0 || T < 0)
    return DYRA_ERR_INVALID_ARG;
  if (p->dtype == DYRA_F32 || p->force_simt) {
    *splits = 1;
    *split_rows = static_cast<int>(T);
    return DYRA_OK;
  }
  dyra::gram_split(T, B, p->d_in, p->k, p->dev.sm_count, splits, split_rows);
  return DYRA_OK;
}

size_t dyra_plan_device_bytes(dyra_plan_t p) {
  if (p == nullptr) return 0;
  return p->factor_bytes + p->cap_Z + p->cap_L + p->cap_TG + p->cap_Tp + p->cap_Ct + p->cap_MD +
         p->cap_Lt + p->cap_P2 + p->cap_TG2 + p->cap_Llo + p->cap_Ctlo + p->cap_Tplo +
         p->cap_Mtmp + 256 +
         (p->bias ? static_cast<size_t>(p->d_out) * elem_size(p->dtype) : 0);
}

}  // extern "C"

// ------------------------------------------------ allocation-free forward ----
// The intermediates of dyra_forward_batched_noalloc live in this array
// instead of the plan's workspace. It is allocated when this file's device
// code is loaded on a device and stays there until the process exits.
static __device__ __align__(256) unsigned char dyra_static_scratch[DYRA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxScratchDevices] = {};
unsigned long long g_scratch_ctx[kMaxScratchDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be
// read). A context torn down and created again gets a new id, and the
// library's device code, the array included, is loaded into it afresh.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(b);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of dyra_static_scratch on `device` (which is current).
// Looked up once per device and context: the first call on a device does the
// lookup, and so does the first call after that device's context was
// destroyed and created again (the array then lives at a new address). Host
// code cannot use the array's name as a device pointer; only this address
// may be handed to kernels.
int static_scratch_address(int device, unsigned char** out) {
  if (device < 0 || device >= kMaxScratchDevices) return DYRA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_addr[device] == nullptr || ctx == 0 || ctx != g_scratch_ctx[device]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, dyra_static_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return DYRA_ERR_CUDA;
    }
    g_scratch_addr[device] = ptr;
    g_scratch_ctx[device] = ctx;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[device]);
  return DYRA_OK;
}

// Carves consecutive 256-byte-aligned pieces out of the fixed array.
struct ScratchCarver {
  unsigned char* base;
  size_t used = 0;
  bool fits = true;
  void* take(size_t bytes) {
    const size_t at = used;
    used += (bytes + 255) & ~static_cast<size_t>(255);
    if (used > DYRA_STATIC_SCRATCH_BYTES) fits = false;
    return base ? base + at : nullptr;
  }
};

}  // namespace

extern "C" int dyra_forward_batched_noalloc(dyra_plan_t p, const void* X, void* Y, int64_t B,
                                            int64_t T, dyra_stream_t stream) {
  if (p == nullptr) return DYRA_ERR_INVALID_ARG;
  if (B < 0 || T < 0) return DYRA_ERR_INVALID_ARG;
  const int64_t N = B * T;
  if (N == 0) return DYRA_OK;
  if (X == nullptr || Y == nullptr) return DYRA_ERR_INVALID_ARG;
  if (N > (static_cast<int64_t>(1) << 31) - 1 || B * static_cast<int64_t>(p->k) > (1 << 30))
    return DYRA_ERR_INVALID_ARG;
  if (!p->loaded) return DYRA_ERR_NOT_LOADED;
  if (p->monarch) return DYRA_ERR_UNSUPPORTED;
  if (!aligned16(X) || !aligned16(Y)) return DYRA_ERR_ALIGNMENT;
  const int k = p->k;
  if (k > 0 && p->lambda == 0.f && T < k) return DYRA_ERR_RANK_DEFICIENT;
  if (k > 0 && p->als_half_steps != 2) return DYRA_ERR_UNSUPPORTED;

  const bool umma = p->dtype == DYRA_BF16 && !p->force_simt;
  const size_t es = elem_size(p->dtype);
  int splits = 1, split_rows = 64;
  if (umma && k > 0) dyra::gram_split(T, B, p->d_in, k, p->dev.sm_count, &splits, &split_rows);

  // Size check first, without touching the device.
  ScratchCarver sizing{nullptr};
  if (umma) {
    sizing.take(static_cast<size_t>(N) * p->r * es);
    if (k > 0) {
      sizing.take(static_cast<size_t>(N) * k * es);
      sizing.take(static_cast<size_t>(B) * k * k * sizeof(float));
      sizing.take(static_cast<size_t>(B) * k * p->d_in * es);
      sizing.take(static_cast<size_t>(B) * k * p->d_out * es);
      sizing.take(factor_bytes(B, k));
      if (use_hilo(p, B, T)) {
        sizing.take(static_cast<size_t>(N) * k * es);
        sizing.take(static_cast<size_t>(B) * k * p->d_out * es);
        sizing.take(static_cast<size_t>(B) * k * p->d_in * es);
      }
    }
  } else {
    sizing.take(static_cast<size_t>(N) * (p->r + k) * es);
    if (k > 0) {
      sizing.take(static_cast<size_t>(B) * k * (p->d_in + k) * sizeof(float));
      sizing.take(static_cast<size_t>(B) * k * p->d_in * es);
      sizing.take(static_cast<size_t>(B) * k * p->d_out * es);
    }
  }
  if (!sizing.fits) return DYRA_ERR_INVALID_ARG;

  DeviceGuard g(p->dev.device);
  if (!g.ok) return DYRA_ERR_CUDA;
  unsigned char* base = nullptr;
  int rc = static_scratch_address(p->dev.device, &base);
  if (rc) return rc;
  ScratchCarver carve{base};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  if (umma) {
    dyra::Bf16Forward a;
    a.d_in = p->d_in;
    a.d_out = p->d_out;
    a.r = p->r;
    a.k = k;
    a.B = B;
    a.T = T;
    a.X = X;
    a.Y = Y;
    a.VPt = p->VPt;
    a.U = p->U;
    a.W_res = p->W_res;
    a.lambda = p->lambda;
    a.weight_only = k == 0;
    a.Z = carve.take(static_cast<size_t>(N) * p->r * es);
    a.L = k > 0 ? carve.take(static_cast<size_t>(N) * k * es) : nullptr;
    a.TG = k > 0 ? static_cast<float*>(carve.take(static_cast<size_t>(B) * k * k * sizeof(float)))
                 : nullptr;
    a.Tp = k > 0 ? carve.take(static_cast<size_t>(B) * k * p->d_in * es) : nullptr;
    a.Ct = k > 0 ? carve.take(static_cast<size_t>(B) * k * p->d_out * es) : nullptr;
    void* fac = k > 0 ? carve.take(factor_bytes(B, k)) : nullptr;
    split_factor_buffer(fac, B, k, &a.MD, &a.counters);
    a.hilo = k > 0 && use_hilo(p, B, T);
    a.Llo = a.hilo ? carve.take(static_cast<size_t>(N) * k * es) : nullptr;
    a.Ctlo = a.hilo ? carve.take(static_cast<size_t>(B) * k * p->d_out * es) : nullptr;
    a.split_t = a.hilo;
    a.Tplo = a.hilo ? carve.take(static_cast<size_t>(B) * k * p->d_in * es) : nullptr;
    a.factor_mode = p->factor_mode;
    a.splits = splits;
    a.split_rows = split_rows;
    a.status = p->status;
    a.stage_events = nullptr;
    a.trace = nullptr;
    a.use_pairs = p->use_pairs;
    a.proj_pair_min_tiles = p->proj_pair_min_tiles;
    a.proj_bn = p->proj_bn;
    a.bias = p->has_bias ? p->bias : nullptr;
    a.alpha = p->alpha;
    a.solver = p->solver;
    a.ns_iters = p->ns_iters;
    rc = dyra::launch_bf16_forward(a, p->dev, s);
  } else if (p->dtype == DYRA_BF16) {
    dyra::SimtForward<__nv_bfloat16> a;
    a.d_in = p->d_in;
    a.d_out = p->d_out;
    a.r = p->r;
    a.k = k;
    a.B = B;
    a.Trows = T;
    a.X = static_cast<const __nv_bfloat16*>(X);
    a.Y = static_cast<__nv_bfloat16*>(Y);
    a.VPt = static_cast<const __nv_bfloat16*>(p->VPt);
    a.U = static_cast<const __nv_bfloat16*>(p->U);
    a.W_res = static_cast<const __nv_bfloat16*>(p->W_res);
    a.lambda = p->lambda;
    a.weight_only = k == 0;
    a.ZL = static_cast<__nv_bfloat16*>(carve.take(static_cast<size_t>(N) * (p->r + k) * es));
    a.TG = k > 0 ? static_cast<float*>(
                       carve.take(static_cast<size_t>(B) * k * (p->d_in + k) * sizeof(float)))
                 : nullptr;
    a.Tp = k > 0 ? static_cast<__nv_bfloat16*>(carve.take(static_cast<size_t>(B) * k * p->d_in * es))
                 : nullptr;
    a.Cm = k > 0 ? static_cast<__nv_bfloat16*>(carve.take(static_cast<size_t>(B) * k * p->d_out * es))
                 : nullptr;
    a.status = p->status;
    a.bias = p->has_bias ? static_cast<const __nv_bfloat16*>(p->bias) : nullptr;
    a.alpha = p->alpha;
    rc = dyra::launch_simt_forward(a, p->dev, s);
  } else {
    dyra::SimtForward<float> a;
    a.d_in = p->d_in;
    a.d_out = p->d_out;
    a.r = p->r;
    a.k = k;
    a.B = B;
    a.Trows = T;
    a.X = static_cast<const float*>(X);
    a.Y = static_cast<float*>(Y);
    a.VPt = static_cast<const float*>(p->VPt);
    a.U = static_cast<const float*>(p->U);
    a.W_res = static_cast<const float*>(p->W_res);
    a.lambda = p->lambda;
    a.weight_only = k == 0;
    a.ZL = static_cast<float*>(carve.take(static_cast<size_t>(N) * (p->r + k) * es));
    a.TG = k > 0 ? static_cast<float*>(
                       carve.take(static_cast<size_t>(B) * k * (p->d_in + k) * sizeof(float)))
                 : nullptr;
    a.Tp = k > 0 ? static_cast<float*>(carve.take(static_cast<size_t>(B) * k * p->d_in * es))
                 : nullptr;
    a.Cm = k > 0 ? static_cast<float*>(carve.take(static_cast<size_t>(B) * k * p->d_out * es))
                 : nullptr;
    a.status = p->status;
    a.bias = p->has_bias ? static_cast<const float*>(p->bias) : nullptr;
    a.alpha = p->alpha;
    rc = dyra::launch_simt_forward(a, p->dev, s);
  }
  if (rc != 0) {
    cudaGetLastError();
    return DYRA_ERR_CUDA;
  }
  return DYRA_OK;
}
