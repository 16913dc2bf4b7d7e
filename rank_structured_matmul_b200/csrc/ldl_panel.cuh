// ldl_panel.cuh - factorisation of the ridge system of the one-step ALS
// correction ("DyRA: Dynamic Residual Approximation for Efficient Matrix
// Multiplication in DNNs", Sec. 2.2 Eq. 5 with footnote 2; Appendix A,
// Algorithm 1, procedure Inference: C = (L^T L + lambda I)^-1 L^T X W_res^T).
//
// Gaussian elimination below the diagonal of [G | I] for a symmetric positive
// definite k x k matrix G (k <= KMAX, padded to KMAX with the identity).
// After k steps the left half's diagonal holds D and the right half holds
// M = Lt^-1, where G = Lt D Lt^T with Lt unit lower triangular, so
// G^-1 = M^T D^-1 M. The two products with M and D^-1 are as accurate as the
// two triangular solves of a Cholesky factorisation and carry no sequential
// dependency. No pivoting: G is positive definite after the ridge; a pivot
// <= 0 or NaN is reported through the return value.
//
// Work split: NT threads (NT / 32 warps) each keep RB rows x CB columns of
// [G | I] in registers. Pivots go in panels of four: the panel's columns and
// rows are broadcast through ping-pong shared buffers, every thread
// eliminates the 4 x 4 pivot block itself and applies a rank-4 update to its
// elements, so there is one barrier per four pivots.
#pragma once

namespace dyra {

constexpr int kLdlPanel = 4;

template <int KMAX>
struct LdlScratch {
  static constexpr int LDG = KMAX + 1;   // odd stride for the staging of G
  float Gs[KMAX * LDG];                  // G + lambda I, padded with the identity
  float colbuf[2][kLdlPanel][KMAX];      // [ping-pong][panel column][row]
  float rowbuf[2][kLdlPanel][2 * KMAX];  // [ping-pong][panel row][column]
};

// Per-instance factor record written by the Gram stage and read by the solve:
// M (KMAX x KMAX, row-major, unit lower), D^-1 (KMAX), a failure flag, padding
// to a 16-byte multiple.
template <int KMAX>
__host__ __device__ constexpr int ldl_record_floats() {
  return KMAX * KMAX + KMAX + 4;
}

// Reciprocal of a pivot (PTX rcp.approx: within one ulp; the factor's own
// rounding error is of the same order).
__device__ __forceinline__ float pivot_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Eliminates sm.Gs (rows and columns beyond k already hold the identity).
// `sync()` is a barrier over the NT participating threads, `tid` this thread's
// index among them. Afterwards `emit_m(i, q, v)` is called for every element
// M[i][q] the thread holds (rows i, columns q of the right half), and
// `emit_d(j, v)` with v = 1 / D[j] for every pivot j (from threads with
// tid < 4, one call per pivot). Returns false if a pivot was <= 0 or not
// finite (the same answer in every thread).
//
// Layout: rows are spread cyclically over the warps (row i = u * NRG + rg) and
// columns over the lanes (column q = v * 32 + lane; v < KMAX / 32 is G, the
// rest is the right half). A panel changes only rows j0 < i < k (the other
// rows get zero multipliers, without branching, so that the rows' dependency
// chains interleave) and, of the 32-column slots, the left ones that reach
// past the panel and the right ones that start at or before its last pivot;
// updates of the other slots are exactly zero and are skipped, warp-uniformly.
template <int KMAX, int NT, class Sync, class EmitM, class EmitD>
__device__ __forceinline__ bool ldl_eliminate(LdlScratch<KMAX>& sm, int k, int tid, Sync sync,
                                              EmitM emit_m, EmitD emit_d) {
  constexpr int NRG = NT / 32;       // row groups (warps)
  constexpr int RB = KMAX / NRG;     // rows of [G | I] per thread
  constexpr int CB = 2 * KMAX / 32;  // column slots per thread
  constexpr int CL = KMAX / 32;      // slots of the left half
  static_assert(NT % 32 == 0 && KMAX % NRG == 0 && KMAX % 32 == 0,
                "thread block does not tile [G | I]");
  constexpr int LDG = LdlScratch<KMAX>::LDG;
  const int rg = tid >> 5, cg = tid & 31;

  float a[RB][CB];
#pragma unroll
  for (int u = 0; u < RB; ++u)
#pragma unroll
    for (int v = 0; v < CB; ++v) {
      const int i = u * NRG + rg, q = v * 32 + cg;
      a[u][v] = q < KMAX ? sm.Gs[i * LDG + q] : (q - KMAX == i ? 1.f : 0.f);
    }
  auto publish = [&](int buf, int j1) {
    // columns j1..j1+3 (every row) and rows j1..j1+3 (every column)
#pragma unroll
    for (int v = 0; v < CL; ++v) {
      const int q = v * 32 + cg;
      if (q >= j1 && q < j1 + kLdlPanel)
#pragma unroll
        for (int u = 0; u < RB; ++u) sm.colbuf[buf][q - j1][u * NRG + rg] = a[u][v];
    }
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      const int i = u * NRG + rg;
      if (i >= j1 && i < j1 + kLdlPanel)
#pragma unroll
        for (int v = 0; v < CB; ++v) sm.rowbuf[buf][i - j1][v * 32 + cg] = a[u][v];
    }
  };
  auto slot_live = [](int v, int j0) {
    return v < CL ? v * 32 + 31 >= j0 + kLdlPanel : (v - CL) * 32 <= j0 + kLdlPanel - 1;
  };
  publish(0, 0);
  sync();
  bool ok = true;
  const int npanel = (k + kLdlPanel - 1) / kLdlPanel;
  for (int pn = 0; pn < npanel; ++pn) {
    const int buf = pn & 1, j0 = pn * kLdlPanel;
    // the panel's pivot rows, at the panel's columns and at this thread's columns
    float Rp[kLdlPanel][kLdlPanel], Ro[kLdlPanel][CB], rinv[kLdlPanel];
#pragma unroll
    for (int r = 0; r < kLdlPanel; ++r) {
#pragma unroll
      for (int c = 0; c < kLdlPanel; ++c) Rp[r][c] = sm.rowbuf[buf][r][j0 + c];
#pragma unroll
      for (int v = 0; v < CB; ++v)
        Ro[r][v] = slot_live(v, j0) ? sm.rowbuf[buf][r][v * 32 + cg] : 0.f;
    }
    // eliminate inside the panel
#pragma unroll
    for (int s2 = 0; s2 < kLdlPanel; ++s2) {
      const float piv = Rp[s2][s2];
      ok = ok && piv > 0.f && isfinite(piv);
      rinv[s2] = pivot_rcp(piv);
      if (tid == s2) emit_d(j0 + s2, rinv[s2]);
#pragma unroll
      for (int r = s2 + 1; r < kLdlPanel; ++r) {
        const float m = Rp[r][s2] * rinv[s2];
#pragma unroll
        for (int c = s2 + 1; c < kLdlPanel; ++c) Rp[r][c] = fmaf(-m, Rp[s2][c], Rp[r][c]);
#pragma unroll
        for (int v = 0; v < CB; ++v)
          if (slot_live(v, j0)) Ro[r][v] = fmaf(-m, Ro[s2][v], Ro[r][v]);
      }
    }
    // multipliers of this thread's rows (zero for rows the panel leaves
    // alone), all rows first so that their dependency chains interleave
    float f[RB][kLdlPanel];
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      const int i = u * NRG + rg;
      const bool live = i > j0 && i < k;
      float cv[kLdlPanel];
#pragma unroll
      for (int c = 0; c < kLdlPanel; ++c) cv[c] = sm.colbuf[buf][c][i];
#pragma unroll
      for (int s2 = 0; s2 < kLdlPanel; ++s2) {
        f[u][s2] = live && i > j0 + s2 ? cv[s2] * rinv[s2] : 0.f;
#pragma unroll
        for (int c = s2 + 1; c < kLdlPanel; ++c) cv[c] = fmaf(-f[u][s2], Rp[s2][c], cv[c]);
      }
    }
    // the rank-4 update, column slot by column slot
#pragma unroll
    for (int v = 0; v < CB; ++v)
      if (slot_live(v, j0))
#pragma unroll
        for (int u = 0; u < RB; ++u)
#pragma unroll
          for (int s2 = 0; s2 < kLdlPanel; ++s2) a[u][v] = fmaf(-f[u][s2], Ro[s2][v], a[u][v]);
    if (j0 + kLdlPanel < k) publish(buf ^ 1, j0 + kLdlPanel);
    sync();
  }
  // pivots past the last panel (identity padding)
  for (int j = npanel * kLdlPanel + tid; j < KMAX; j += NT) emit_d(j, 1.f);
#pragma unroll
  for (int u = 0; u < RB; ++u)
#pragma unroll
    for (int v = CL; v < CB; ++v) emit_m(u * NRG + rg, (v - CL) * 32 + cg, a[u][v]);
  return ok;
}

}  // namespace dyra
