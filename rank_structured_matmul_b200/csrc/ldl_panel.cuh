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
// The elimination is blocked (16 x 16 blocks, see ldl_blocked below): the
// sequential part is one warp's register-shuffle factorisation of each
// diagonal block; everything else is small block products spread over the
// warps.
#pragma once

namespace dyra {

// Per-instance factor record, written by the instance's factoring solve block
// and read by the others: G^-1 (KMAX x KMAX, row-major), a failure flag,
// padding to a 16-byte multiple.
template <int KMAX>
__host__ __device__ constexpr int ldl_record_floats() {
  return KMAX * KMAX + 4;
}

// Reciprocal of a pivot (PTX rcp.approx: within one ulp; the factor's own
// rounding error is of the same order).
__device__ __forceinline__ float pivot_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Blocked form of the same elimination, for KMAX = 32 or 64: 16 x 16 blocks.
// For each block column J:
//   1. one warp factors the diagonal block A_JJ = L_JJ D_J L_JJ^T by
//      eliminating [A_JJ | I] with register shuffles (no barrier), giving
//      M_JJ = L_JJ^-1 and D_J;
//   2. panel: W_IJ = A_IJ M_JJ^T and L_IJ = W_IJ D_J^-1 for I > J;
//   3. trailing update: A_IK -= L_IJ W_KJ^T for J < K <= I.
// Then M = Lt^-1 block by block: N_IP = -M_II L_IP, and by increasing
// distance M_IK = sum over K <= P < I of N_IP M_PK. Each step is the
// unblocked elimination's arithmetic regrouped; there is no pivoting and no
// explicit inverse of anything but unit triangular blocks.
template <int KMAX>
struct LdlBlockScratch {
  static constexpr int LD = KMAX + 1;  // odd stride: conflict-free column access
  float Gs[KMAX * LD];                 // G + lambda I (identity padded); L below the diagonal blocks
  float Mb[KMAX * LD];                 // M = Lt^-1
  float Wb[KMAX * LD];                 // W_IJ, then N_IP
  float dinv[KMAX];                    // 1 / D
  int bad;
};

// One warp: factor the 16 x 16 block at (j0, j0) of sm.Gs. Lanes 0..15 own its
// rows; writes M_JJ into sm.Mb and calls emit_d(j0 + p, 1 / D[p]). Returns
// false if a pivot was <= 0 or not finite (the same answer in every lane).
template <int KMAX, class EmitD>
__device__ __forceinline__ bool ldl_leaf16(LdlBlockScratch<KMAX>& sm, int j0, int lane,
                                           EmitD emit_d) {
  constexpr int LD = LdlBlockScratch<KMAX>::LD;
  const int i = lane & 15;
  float a[16], m[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    a[q] = sm.Gs[(j0 + i) * LD + j0 + q];
    m[q] = q == i ? 1.f : 0.f;
  }
  bool ok = true;
  float dv = 1.f;  // this lane's 1 / D
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    // row p (pivot and the rest) first: the shuffles do not wait on this
    // pivot's arithmetic, so they are all in flight at once
    float ra[16], rm[16];
#pragma unroll
    for (int q = p; q < 16; ++q) ra[q] = __shfl_sync(0xffffffffu, a[q], p);
#pragma unroll
    for (int q = 0; q <= p; ++q) rm[q] = __shfl_sync(0xffffffffu, m[q], p);
    const float d = ra[p];
    ok = ok && d > 0.f && isfinite(d);
    const float r = pivot_rcp(d);
    if (i == p) dv = r;
    const float f = i > p ? a[p] * r : 0.f;
#pragma unroll
    for (int q = p + 1; q < 16; ++q) a[q] = fmaf(-f, ra[q], a[q]);
#pragma unroll
    for (int q = 0; q <= p; ++q) m[q] = fmaf(-f, rm[q], m[q]);
  }
  if (lane < 16) {
    sm.dinv[j0 + i] = dv;
    emit_d(j0 + i, dv);
  }
  if (lane < 16)
#pragma unroll
    for (int q = 0; q < 16; ++q) sm.Mb[(j0 + i) * LD + j0 + q] = m[q];
  return ok;
}

// One warp, one 16 x 16 output block: acc[cc] += sum_q A[r][q] * B(q, c) with
// r = lane % 16 and c = 8 * (lane / 16) + cc, where B(q, c) = B[c][q] (BT) or
// B[q][c]. A and B point at the blocks' first elements, row stride LD. The
// lane keeps its row of A in registers; B's values are shared (broadcast) by
// the lanes of a half-warp.
template <int LD, bool BT>
__device__ __forceinline__ void block16_mma(const float* A, const float* B, int lane,
                                            float acc[8]) {
  const int r = lane & 15, h = lane >> 4;
  float a[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) a[q] = A[r * LD + q];
#pragma unroll
  for (int q = 0; q < 16; ++q)
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const int c = 8 * h + cc;
      acc[cc] = fmaf(a[q], BT ? B[c * LD + q] : B[q * LD + c], acc[cc]);
    }
}

// Factor sm.Gs (KMAX x KMAX, rows and columns beyond k already the identity)
// with NT threads; `sync()` is a barrier over them. Afterwards emit_m(i, q, v)
// is called for every element of M = Lt^-1 (each once, by some thread) and
// emit_d(j, v) with v = 1 / D[j] for every j < KMAX. Returns false if a pivot
// was <= 0 or not finite (the same answer in every thread). The block
// products run one 16 x 16 block per warp.
// ts (optional): a timeline row; thread 0 stamps %globaltimer into ts[2J] after
// block column J's leaf and ts[2J + 1] after its trailing update, ts[8] after
// the assembly of M and ts[9] after the emits.
template <int KMAX, int NT, class Sync, class EmitM, class EmitD>
__device__ __forceinline__ bool ldl_blocked(LdlBlockScratch<KMAX>& sm, int k, int tid, Sync sync,
                                            EmitM emit_m, EmitD emit_d,
                                            unsigned long long* ts = nullptr) {
  auto stamp = [&](int slot) {
    if (ts && tid == 0) {
      unsigned long long t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)::"memory");
      ts[slot] = t;
    }
  };
  static_assert(KMAX == 32 || KMAX == 64, "blocked LDL needs KMAX 32 or 64");
  static_assert(NT % 32 == 0, "whole warps");
  constexpr int NB = KMAX / 16;
  constexpr int NW = NT / 32;
  constexpr int LD = LdlBlockScratch<KMAX>::LD;
  const int warp = tid >> 5, lane = tid & 31;
  const int r16 = lane & 15, h8 = 8 * (lane >> 4);
  const int nbk = (k + 15) / 16;  // block columns with real pivots; the rest is identity
  if (tid == 0) sm.bad = 0;
  // M starts as zero above the diagonal blocks (the blocks below are written by
  // the assembly, the diagonal blocks by the leaves)
  for (int e = tid; e < KMAX * KMAX; e += NT) {
    const int r = e / KMAX, c = e % KMAX;
    if (c / 16 > r / 16) sm.Mb[r * LD + c] = 0.f;
  }
  for (int J = 0; J < NB; ++J) {
    const int j0 = 16 * J;
    if (J >= nbk) {  // identity padding: M_JJ = I, D = 1
      for (int e = tid; e < 256; e += NT) {
        const int r = e >> 4, c = e & 15;
        sm.Mb[(j0 + r) * LD + j0 + c] = r == c ? 1.f : 0.f;
        if (r == c) {
          sm.dinv[j0 + r] = 1.f;
          emit_d(j0 + r, 1.f);
        }
      }
      continue;
    }
    if (warp == 0) {
      const bool ok = ldl_leaf16<KMAX>(sm, j0, lane, emit_d);
      if (!ok && lane == 0) sm.bad = 1;
    }
    sync();
    stamp(2 * J);
    if (J + 1 == NB) break;
    // panel: W_IJ = A_IJ M_JJ^T (into Wb) and L_IJ = W_IJ D_J^-1 (over A_IJ)
    for (int I = J + 1 + warp; I < NB; I += NW) {
      float acc[8] = {};
      block16_mma<LD, true>(&sm.Gs[(16 * I) * LD + j0], &sm.Mb[j0 * LD + j0], lane, acc);
      __syncwarp();  // every lane has read its row of A_IJ
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const int r = 16 * I + r16, c = j0 + h8 + cc;
        sm.Wb[r * LD + c] = acc[cc];
        sm.Gs[r * LD + c] = acc[cc] * sm.dinv[c];
      }
    }
    sync();
    // trailing: A_IK -= L_IJ W_KJ^T for J < K <= I (diagonal blocks in full)
    {
      const int nt = NB - 1 - J;  // trailing block rows
      for (int t = warp; t < nt * (nt + 1) / 2; t += NW) {
        int I = 0, K = 0, cnt = t;  // t-th lower block (I, K), row-major
        for (int ii = 0; ii < nt; ++ii) {
          if (cnt <= ii) {
            I = J + 1 + ii;
            K = J + 1 + cnt;
            break;
          }
          cnt -= ii + 1;
        }
        float acc[8] = {};
        block16_mma<LD, true>(&sm.Gs[(16 * I) * LD + j0], &sm.Wb[(16 * K) * LD + j0], lane, acc);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          float& g = sm.Gs[(16 * I + r16) * LD + 16 * K + h8 + cc];
          g -= acc[cc];
        }
      }
    }
    sync();
    stamp(2 * J + 1);
  }
  sync();  // identity-padded blocks above are written without a barrier of their own
  // M below the diagonal blocks: N_IP = -M_II L_IP (into Wb), then by distance
  // M_IK = sum_{K <= P < I} N_IP M_PK
  for (int t = warp; t < NB * (NB - 1) / 2; t += NW) {
    int I = 0, P = 0, cnt = t;  // t-th strictly lower block (I, P)
    for (int ii = 1; ii < NB; ++ii) {
      if (cnt < ii) {
        I = ii;
        P = cnt;
        break;
      }
      cnt -= ii;
    }
    float acc[8] = {};
    block16_mma<LD, false>(&sm.Mb[(16 * I) * LD + 16 * I], &sm.Gs[(16 * I) * LD + 16 * P], lane,
                           acc);
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) sm.Wb[(16 * I + r16) * LD + 16 * P + h8 + cc] = -acc[cc];
  }
  sync();
  for (int dist = 1; dist < NB; ++dist) {
    for (int K = warp; K + dist < NB; K += NW) {
      const int I = K + dist;
      float acc[8] = {};
      for (int P = K; P < I; ++P)
        block16_mma<LD, false>(&sm.Wb[(16 * I) * LD + 16 * P], &sm.Mb[(16 * P) * LD + 16 * K],
                               lane, acc);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) sm.Mb[(16 * I + r16) * LD + 16 * K + h8 + cc] = acc[cc];
    }
    sync();
  }
  stamp(8);
  for (int e = tid; e < KMAX * KMAX; e += NT) emit_m(e / KMAX, e % KMAX, sm.Mb[(e / KMAX) * LD + e % KMAX]);
  stamp(9);
  return sm.bad == 0;
}

}  // namespace dyra
