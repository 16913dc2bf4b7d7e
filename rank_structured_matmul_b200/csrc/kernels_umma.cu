// kernels_umma.cu - the bf16 DyRA forward on tcgen05 tensor cores.
//
// Method: "DyRA: Dynamic Residual Approximation for Efficient Matrix
// Multiplication in DNNs", Appendix A, Algorithm 1, procedure Inference, with
// the correction fitted per batch instance (Sec. 2.4). Letters: static rank r,
// correction rank k, Y = X W^T with W = d_out x d_in.
//
// Four tensor-core GEMMs and one small solve, stream-ordered:
//   proj    [Z | L] = X [V | P]                     static part and left factor, Eq. 7
//   gram    per instance b: T_b = L_b^T X_b (bf16), G_b = L_b^T L_b (fp32)
//   rfactor Q^T = W_res T^T, all instances at once
//   solve   L~_b = L_b (G_b + lambda I)^-1, beside rfactor (kernels_simt.cu)
//   out     Y = Z U^T + sum_b mask_b(L~) Q_b, one TMEM accumulation (the output step)
// L~_b Q_b = L_b C_b with C_b the paper's R^(1) for instance b, the right factor
// (G_b + lambda I)^-1 (L_b^T X_b) W_res^T: the same product, grouped so that
// the large GEMM needs no factorisation.
//
// Storage bf16, accumulation fp32 in tensor memory. Every operand tile is
// brought in by TMA with 128-byte swizzling (64 bf16 per row); tiles that run
// past a tensor's edge are zero-filled by TMA, which also masks instance
// boundaries: L and X are addressed as 3-D (k or d_in, T, B) tensors, so rows
// outside the instance read as zero.
#include <algorithm>
#include <cstdio>

#include "internal.h"
#include "ldl_panel.cuh"
#include "umma_gemm.cuh"
#include "umma_gemm_pair.cuh"

namespace dyra {

using namespace sm100;

namespace {

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int ks) {
  // K-major, 128-byte swizzle: rows of 64 bf16, 8-row atoms 1024 bytes apart;
  // the k-th group of 16 elements starts 32 bytes further into each row.
  return smem_desc(base + static_cast<uint32_t>(ks) * 32u, 16u, 1024u, kLayoutSw128);
}

__device__ __forceinline__ float f32(uint32_t u) { return __uint_as_float(u); }

// Split-K reductions over distributed shared memory: float4 items off[u] of
// the partials of cluster ranks ks .. ks + NJ - 1, all loads in flight at once.
template <int NJ>
__device__ __forceinline__ void load_partials(float4 (&v)[4][4], uint32_t stage_u32, int ks,
                                              const uint32_t (&off)[4]) {
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const uint32_t base = mapa_shared(stage_u32, static_cast<uint32_t>(ks + j));
#pragma unroll
    for (int u = 0; u < 4; ++u) v[j][u] = ld_shared_cluster_v4(base + 16u * off[u]);
  }
}
// Loads the min(4, S - ks) partials from rank ks on (each partial read once:
// the reads are bound by the bandwidth of distributed shared memory).
__device__ __forceinline__ void load_partials_from(float4 (&v)[4][4], uint32_t stage_u32, int ks,
                                                   int S, const uint32_t (&off)[4]) {
  switch (min(4, S - ks)) {
    case 4: load_partials<4>(v, stage_u32, ks, off); break;
    case 3: load_partials<3>(v, stage_u32, ks, off); break;
    case 2: load_partials<2>(v, stage_u32, ks, off); break;
    default: load_partials<1>(v, stage_u32, ks, off); break;
  }
}

// Write eight fp32 accumulator values as one 16-byte bf16 vector.
__device__ __forceinline__ void store8_bf16(void* dst, const uint32_t (&v)[32], int g) {
  st_global_v4(dst, pack_bf16x2(f32(v[8 * g + 0]), f32(v[8 * g + 1])),
               pack_bf16x2(f32(v[8 * g + 2]), f32(v[8 * g + 3])),
               pack_bf16x2(f32(v[8 * g + 4]), f32(v[8 * g + 5])),
               pack_bf16x2(f32(v[8 * g + 6]), f32(v[8 * g + 7])));
}

__device__ __forceinline__ int ceil_div_dev(int a, int b) { return (a + b - 1) / b; }

// Epilogue helper: writes one 128 x 64 box of the accumulator (TMEM columns
// col0 .. col0+63 of this thread's row) as bf16 through a 128-byte-swizzled
// shared-memory box and a TMA store at (x, y) of `tmap`. Two boxes rotate: a
// box is rewritten only after the store issued two boxes earlier has read it.
// All 128 epilogue threads call it; thread 0 issues the stores. With `bias`
// (ncols entries, ncols a multiple of 8) bias[x + j] is added to column j of
// the box in fp32 before the rounding; columns at or beyond ncols read none.
constexpr uint32_t kStoreBoxBytes = 128u * 128u;  // 128 rows x 64 bf16
constexpr uint32_t kStoreBoxes = 2;

// With LO set, the box receives the low part of each value instead,
// bf16(v - bf16(v)): the two boxes together carry v to about 16 bits. BIAS
// compiles the bias add in (the callers without one keep the plain loop).
template <bool LO = false, bool BIAS = false>
__device__ __forceinline__ void store_box_bf16(uint32_t tacc, int col0, const void* tmap, int x,
                                               int y, EpiCtx& e,
                                               const __nv_bfloat16* bias = nullptr,
                                               int ncols = 0) {
  const uint32_t buf = e.counter % kStoreBoxes;
  ++e.counter;
  // the box's 64 bias values (8 columns per load, all inside or all beyond
  // ncols) are loaded first, so that their latency passes during the TMEM
  // loads and the wait for the store buffer
  uint4 bq[BIAS ? 8 : 1];
  if constexpr (BIAS) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = x + j * 8;
      bq[j] = c < ncols ? __ldg(reinterpret_cast<const uint4*>(bias + c)) : make_uint4(0, 0, 0, 0);
    }
  }
  // both TMEM loads in flight before one wait, and during the wait for the
  // store buffer
  uint32_t vv[2][32];
  tmem_ld_32x32b_x32(tacc + col0, vv[0]);
  tmem_ld_32x32b_x32(tacc + col0 + 32, vv[1]);
  if (e.tid == 0) tma_store_wait_read<kStoreBoxes - 1>();
  named_bar_sync(1, 128);
  uint8_t* sbuf = e.smem + buf * kStoreBoxBytes;
  tmem_ld_wait();
  if constexpr (BIAS) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const uint4& b8 = bq[half * 4 + ch];
        const uint32_t w[4] = {b8.x, b8.y, b8.z, b8.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t& v0 = vv[half][8 * ch + 2 * j];
          uint32_t& v1 = vv[half][8 * ch + 2 * j + 1];
          v0 = __float_as_uint(f32(v0) + __uint_as_float(w[j] << 16));
          v1 = __float_as_uint(f32(v1) + __uint_as_float(w[j] & 0xffff0000u));
        }
      }
    }
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      const int chunk = half * 4 + ch;
      const uint32_t off =
          static_cast<uint32_t>(e.row) * 128u + static_cast<uint32_t>((chunk ^ (e.row & 7)) * 16);
      auto val = [&](int c) {
        const float v = f32(vv[half][8 * ch + c]);
        return LO ? v - __bfloat162float(__float2bfloat16_rn(v)) : v;
      };
      uint4 q;
      q.x = pack_bf16x2(val(0), val(1));
      q.y = pack_bf16x2(val(2), val(3));
      q.z = pack_bf16x2(val(4), val(5));
      q.w = pack_bf16x2(val(6), val(7));
      *reinterpret_cast<uint4*>(sbuf + off) = q;
    }
  }
  fence_async_shared();
  named_bar_sync(1, 128);
  if (e.tid == 0) {
    tma_store_2d(tmap, e.smem_u32 + buf * kStoreBoxBytes, x, y);
    tma_store_commit();
  }
}


__device__ __forceinline__ void store_drain(EpiCtx& e) {
  if (e.tid == 0) tma_store_wait_all();
}

}  // namespace

// =================================================================== proj ====
// [Z | L] = X . [V | P]: A = X (K-major), B = [V|P]^T (K-major). X is read
// from HBM once; the n-tiles of one m-tile run on neighbouring CTAs and share
// it through L2.
struct ProjPolicy {
  struct Params {
    GemmCommon c;
    CUtensorMap tmX;  // (d_in, N), box (64, 128)
    CUtensorMap tmW;  // (d_in, r+k), box (64, bn)
    CUtensorMap tmZ;  // (r, N), box (64, 128), store
    CUtensorMap tmL;  // (k, N), box (64, 128), store (a 64-column box covers k <= 64 columns)
    int N, d_in, r, k, bn, n_tiles_n;
    int tma_store;    // r % 64 == 0 and k <= 64: every 64-column box is all Z or all L
    __nv_bfloat16* Z;
    __nv_bfloat16* L;
    int* cnt;         // the per-instance flags or counters of later stages, cleared here (or nullptr)
    int ncnt;
    // Split-K for skinny N (ksplit > 1): the ksplit CTAs of output tile
    // `base` form one cluster; CTA ks takes k-iterations [ks * kper,
    // (ks + 1) * kper) and leaves its fp32 partial tile in its own shared
    // memory; after a cluster barrier each CTA sums the partials of its slice
    // of rows over distributed shared memory, in split order, and stores Z
    // and L. One tile per CTA.
    int ksplit, kper;
  };
  struct Tile {
    int m0, n0, ks, base;
  };
  static constexpr uint32_t kEpiSmemBytes = kStoreBoxes * kStoreBoxBytes;

  static __device__ __forceinline__ void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmX);
    tma_prefetch_desc(&p.tmW);
    if (p.tma_store) {
      tma_prefetch_desc(&p.tmZ);
      if (p.k > 0) tma_prefetch_desc(&p.tmL);
    }
  }
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    t.base = tile / p.ksplit;
    t.ks = tile - t.base * p.ksplit;
    t.m0 = (t.base / p.n_tiles_n) * 128;
    t.n0 = (t.base % p.n_tiles_n) * p.bn;
  }
  static __device__ __forceinline__ int kiters(const Params& p, const Tile& t) {
    const int total = ceil_div_dev(p.d_in, 64);
    return p.ksplit > 1 ? min(p.kper, total - t.ks * p.kper) : total;
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar) {
    load_early(p, t, it, sa, sb, bar);
    load_late(p, t, it, sa, sb, bar);
  }
  // [V | P]^T is a loaded weight, ready before any grid of the forward runs;
  // X may be the output of the grid just before this one.
  static constexpr bool kEarly = true;
  static __device__ __forceinline__ void load_early(const Params& p, const Tile& t, int it,
                                                    uint32_t, uint32_t sb, uint32_t bar) {
    tma_load_2d(sb, &p.tmW, bar, (t.ks * p.kper + it) * 64, t.n0);
  }
  static __device__ __forceinline__ void load_late(const Params& p, const Tile& t, int it,
                                                   uint32_t sa, uint32_t, uint32_t bar) {
    tma_load_2d(sa, &p.tmX, bar, (t.ks * p.kper + it) * 64, t.m0);
  }
  static __device__ __forceinline__ int ksteps(const Params& p, const Tile& t, int it) {
    return min(4, ceil_div_dev(p.d_in - (t.ks * p.kper + it) * 64, 16));
  }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    return kmajor_desc(a, ks);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params&, uint32_t b, int ks) {
    return kmajor_desc(b, ks);
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    // The Gram stage starts after this grid completes, so clearing its
    // counters here makes every forward start from zero.
    if (p.cnt && t.m0 == 0 && t.n0 == 0)
      for (int i = e.tid; i < p.ncnt; i += 128) p.cnt[i] = 0;
    const int rk = p.r + p.k;
    if (p.ksplit > 1) {
      split_epilogue(p, t, tacc, e);
      return;
    }
    if (p.tma_store) {
      for (int bx = 0; bx < p.bn / 64; ++bx) {
        const int col = t.n0 + bx * 64;
        if (col >= rk) break;
        if (col < p.r)
          store_box_bf16(tacc, bx * 64, &p.tmZ, col, t.m0, e);
        else
          store_box_bf16(tacc, bx * 64, &p.tmL, col - p.r, t.m0, e);
      }
      return;
    }
    const int grow = t.m0 + e.row;
    for (int cc = 0; cc < p.bn; cc += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + cc, v);
      tmem_ld_wait();
      if (grow < p.N) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = t.n0 + cc + 8 * g;
          if (col < rk && cc + 8 * g < p.bn) {  // the last 32 columns may pass the tile
            const bool z = col < p.r;
            const size_t at = z ? static_cast<size_t>(grow) * p.r + col
                                : static_cast<size_t>(grow) * p.k + (col - p.r);
            if (!in_bounds(p.c.status, at, 8, static_cast<size_t>(p.N) * (z ? p.r : p.k)))
              continue;
            store8_bf16(z ? static_cast<void*>(p.Z + at) : static_cast<void*>(p.L + at), v, g);
          }
        }
      }
    }
  }
  // Split-K, first half: the partial tile into this CTA's operand stages,
  // column-major in float4 units ([c4][row]: a warp writes 512 contiguous
  // bytes, and the reads below are conflict-free too).
  static __device__ __forceinline__ void split_epilogue(const Params& p, const Tile&,
                                                        uint32_t tacc, EpiCtx& e) {
    float4* part = reinterpret_cast<float4*>(e.stage);
    for (int cc = 0; cc < p.bn; cc += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + cc, v);
      tmem_ld_wait();
#pragma unroll
      for (int g = 0; g < 8; ++g)
        part[(cc / 4 + g) * 128 + e.row] =
            make_float4(f32(v[4 * g]), f32(v[4 * g + 1]), f32(v[4 * g + 2]), f32(v[4 * g + 3]));
    }
    if (e.tr && e.tid == 0) e.tr[kTrSplitWritten] = globaltimer_ns();
  }
  static __device__ __forceinline__ bool cluster_finish(const Params& p) { return p.ksplit > 1; }
  // Split-K, second half (after the cluster barrier): this CTA's slice of
  // rows, summed over the cluster's partials in split order.
  static __device__ __noinline__ void finish(const Params& p, int tid, uint32_t stage_u32,
                                             unsigned long long* tr) {
    if (tr && tid == 0) tr[kTrSplitArrived] = globaltimer_ns();
    const int ks_me = static_cast<int>(cluster_ctarank());
    Tile t;
    decode(p, static_cast<int>(blockIdx.x), t);
    // this CTA's slice of the tile's rows, cut at the last row of X, and the
    // tile's columns inside [Z | L]: the rest is never stored, and the reads
    // of the partials are bound by the bandwidth of distributed shared memory
    const int rk = p.r + p.k;
    const int c4n = min(p.bn / 4, max(0, (rk - t.n0 + 3) / 4));
    const int rs = (128 + p.ksplit - 1) / p.ksplit;
    const int row0 = ks_me * rs;
    const int nrows = max(0, min(min(128, row0 + rs), p.N - t.m0) - row0);
    const int nitems = nrows * c4n;
    for (int i0 = tid; i0 < nitems; i0 += 4 * 128) {
      uint32_t off[4];
      bool valid[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = i0 + u * 128;
        valid[u] = it < nitems;
        const int c4 = valid[u] ? it / nrows : 0;
        const int row = valid[u] ? row0 + (it - c4 * nrows) : row0;
        off[u] = static_cast<uint32_t>(c4 * 128 + row);
      }
      float4 acc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int ks = 0; ks < p.ksplit; ks += 4) {
        float4 v[4][4];
        load_partials_from(v, stage_u32, ks, p.ksplit, off);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (ks + j < p.ksplit)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              acc[u].x += v[j][u].x;
              acc[u].y += v[j][u].y;
              acc[u].z += v[j][u].z;
              acc[u].w += v[j][u].w;
            }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (!valid[u]) continue;
        const int c4 = static_cast<int>(off[u]) / 128, row = static_cast<int>(off[u]) - c4 * 128;
        const int grow = t.m0 + row, col = t.n0 + 4 * c4;
        if (grow >= p.N || col >= rk) continue;
        const bool z = col < p.r;
        const size_t at = z ? static_cast<size_t>(grow) * p.r + col
                            : static_cast<size_t>(grow) * p.k + (col - p.r);
        if (!in_bounds(p.c.status, at, 4, static_cast<size_t>(p.N) * (z ? p.r : p.k))) continue;
        __nv_bfloat16* dst = (z ? p.Z : p.L) + at;
        uint2 w;
        w.x = pack_bf16x2(acc[u].x, acc[u].y);
        w.y = pack_bf16x2(acc[u].z, acc[u].w);
        *reinterpret_cast<uint2*>(dst) = w;
      }
    }
    if (tr && tid == 0) tr[kTrSplitReduced] = globaltimer_ns();
  }
  static __device__ __forceinline__ void epilogue_drain(const Params& p, EpiCtx& e) {
    if (p.tma_store && p.ksplit <= 1) store_drain(e);
  }
};

// =================================================================== gram ====
// For every instance b: D = [X_b | L_b]^T L_b, i.e. T_b^T (d_in x k) and G_b
// (k x k), written as T[b*k + i][j] = T_b[i][j] (bf16, the next GEMM's
// K-major operand) and G[b][i][i'] (fp32, for the factorisation). Both
// operands are MN-major (the reduction runs over rows of X and L). With S > 1
// row splits the S CTAs of one (m-tile, instance) form a cluster: each leaves
// its fp32 partial tile in its own operand stages and, after a cluster
// barrier, sums one slice of rows over all S partials through distributed
// shared memory (split-K, as in the projection).
// kAls: the options the L update of further ALS iterations needs (an X view
// shared by every instance, and T and G in fp32 as B x k x (d_in + k)); the
// one-step layer's Gram stage is compiled without them. kLo: T is also stored
// as its bf16 rounding errors (Tlo, the split T of the compensated correction).
template <bool kAls, bool kLo>
struct GramPolicyT {
  struct Params {
    GemmCommon c;
    CUtensorMap tmX;   // (d_in, T, B), box (64, 64, 1), 128B swizzle
    CUtensorMap tmLa;  // (k, T, B),    box (64, 64, 1), 128B swizzle   (A role)
    CUtensorMap tmLb;  // (k, T, B),    box (w, 64, 1),  w*2-byte swizzle (B role)
    int d_in, k, kpad, w, nbox_b, T, B, S, Ts, mtx, mt_total;
    uint32_t b_layout;
    // 1: the X view holds one instance that every instance b reads (its third
    // coordinate is 0 for all b), e.g. W_res for the L update of more ALS
    // iterations, where "T" counts d_out rows
    int x_inst_fixed;
    __nv_bfloat16* Tb;  // (B*k) x d_in
    __nv_bfloat16* Tlo;  // (B*k) x d_in: the bf16 rounding errors of Tb (kLo)
    float* G;           // B x k x k
    // when set, T and G go here instead, in fp32, as B x k x (d_in + k):
    // row i of instance b holds (L_b^T X_b)[i][0..d_in) then (L_b^T L_b)[i][0..k)
    float* TGf;
  };
  struct Tile {
    int mt, b, s, t0, t1;
  };
  static constexpr uint32_t kEpiSmemBytes = 0;

  static __device__ __forceinline__ void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmX);
    tma_prefetch_desc(&p.tmLa);
    tma_prefetch_desc(&p.tmLb);
  }
  // The S splits of one output tile are neighbours (one cluster); tiles of G
  // (the m-tiles over L's columns) come first.
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    const int g = tile / p.S;
    t.s = tile - g * p.S;
    const int mtl = p.mt_total - p.mtx;
    const int ng = mtl * p.B;
    if (g < ng) {
      t.mt = p.mtx + g % mtl;
      t.b = g / mtl;
    } else {
      t.mt = (g - ng) % p.mtx;
      t.b = (g - ng) / p.mtx;
    }
    t.t0 = t.s * p.Ts;
    t.t1 = min(p.T, t.t0 + p.Ts);
  }
  static __device__ __forceinline__ int kiters(const Params&, const Tile& t) {
    return ceil_div_dev(t.t1 - t.t0, 64);
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar) {
    const int row = t.t0 + it * 64;
    if (t.mt < p.mtx) {
      const int j0 = t.mt * 128;
      const int bx = kAls && p.x_inst_fixed ? 0 : t.b;
      tma_load_3d(sa, &p.tmX, bar, j0, row, bx);
      tma_load_3d(sa + 8192u, &p.tmX, bar, j0 + 64, row, bx);
    } else {
      const int i0 = (t.mt - p.mtx) * 128;
      tma_load_3d(sa, &p.tmLa, bar, i0, row, t.b);
      tma_load_3d(sa + 8192u, &p.tmLa, bar, i0 + 64, row, t.b);
    }
    const uint32_t box_b = static_cast<uint32_t>(p.w) * 2u * 64u;
    for (int q = 0; q < p.nbox_b; ++q) tma_load_3d(sb + q * box_b, &p.tmLb, bar, 64 * q, row, t.b);
  }
  static __device__ __forceinline__ int ksteps(const Params&, const Tile&, int) { return 4; }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    // MN-major, 128-byte swizzle: 64 elements of M per 128-byte row, 8 K-rows
    // per 1024-byte atom (SBO), the second 64-wide M block 8 KB away (LBO).
    return smem_desc(a + static_cast<uint32_t>(ks) * 2048u, 8192u, 1024u, kLayoutSw128);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params& p, uint32_t b, int ks) {
    const uint32_t rb = static_cast<uint32_t>(p.w) * 2u;  // bytes per K-row of one block
    return smem_desc(b + static_cast<uint32_t>(ks) * 16u * rb, 64u * rb, 8u * rb, p.b_layout);
  }
  // Stores v[0..n) = D[row][i0 .. i0+n) of tile t (tile row `row`): into T
  // (bf16) for the m-tiles over X, into G (fp32) for the one over L.
  template <int n>
  static __device__ __forceinline__ void store_row(const Params& p, const Tile& t, int row, int i0,
                                                   const float (&v)[n]) {
    if (kAls && p.TGf != nullptr) {
      const int J = p.d_in + p.k;
      float* inst = p.TGf + static_cast<size_t>(t.b) * p.k * J;
      int col;  // column of instance b's k x J block that this thread's row feeds
      if (t.mt < p.mtx) {
        col = t.mt * 128 + row;
        if (col >= p.d_in) return;
      } else {
        const int i2 = (t.mt - p.mtx) * 128 + row;
        if (i2 >= p.k) return;
        col = p.d_in + i2;
      }
      const size_t extent = static_cast<size_t>(p.B) * p.k * J;
#pragma unroll
      for (int u = 0; u < n; ++u)
        if (i0 + u < p.k &&
            in_bounds(p.c.status, (inst - p.TGf) + static_cast<size_t>(i0 + u) * J + col, 1,
                      extent))
          inst[static_cast<size_t>(i0 + u) * J + col] = v[u];
      return;
    }
    if (t.mt < p.mtx) {
      const int j = t.mt * 128 + row;
      if (j >= p.d_in) return;
      const size_t off = static_cast<size_t>(t.b) * p.k * p.d_in + j;
      __nv_bfloat16* dst = p.Tb + off;
      const size_t extent = static_cast<size_t>(p.B) * p.k * p.d_in;
#pragma unroll
      for (int u = 0; u < n; ++u)
        if (i0 + u < p.k &&
            in_bounds(p.c.status, off + static_cast<size_t>(i0 + u) * p.d_in, 1, extent)) {
          const __nv_bfloat16 h = __float2bfloat16_rn(v[u]);
          dst[static_cast<size_t>(i0 + u) * p.d_in] = h;
          if (kLo)
            p.Tlo[off + static_cast<size_t>(i0 + u) * p.d_in] =
                __float2bfloat16_rn(v[u] - __bfloat162float(h));
        }
    } else {
      const int i2 = (t.mt - p.mtx) * 128 + row;
      if (i2 >= p.k) return;
      float* dst = p.G + static_cast<size_t>(t.b) * p.k * p.k + i2;
      const size_t extent = static_cast<size_t>(p.B) * p.k * p.k;
#pragma unroll
      for (int u = 0; u < n; ++u)
        if (i0 + u < p.k &&
            in_bounds(p.c.status, (dst - p.G) + static_cast<size_t>(i0 + u) * p.k, 1, extent))
          dst[static_cast<size_t>(i0 + u) * p.k] = v[u];
    }
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    if (p.S > 1) {
      // the partial tile into this CTA's operand stages, [c4][row] float4s
      float4* part = reinterpret_cast<float4*>(e.stage);
      for (int cc = 0; cc < p.kpad; cc += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tacc + cc, v);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 8; ++g)
          part[(cc / 4 + g) * 128 + e.row] =
              make_float4(f32(v[4 * g]), f32(v[4 * g + 1]), f32(v[4 * g + 2]), f32(v[4 * g + 3]));
      }
      if (e.tr && e.tid == 0) e.tr[kTrSplitWritten] = globaltimer_ns();
      return;
    }
    for (int cc = 0; cc < p.kpad; cc += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + cc, v);
      tmem_ld_wait();
      float f[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) f[jj] = f32(v[jj]);
      store_row(p, t, e.row, cc, f);
    }
  }
  static __device__ __forceinline__ bool cluster_finish(const Params& p) { return p.S > 1; }
  // After the cluster barrier: this CTA's slice of rows, summed over the
  // cluster's partials in split order.
  static __device__ __noinline__ void finish(const Params& p, int tid, uint32_t stage_u32,
                                             unsigned long long* tr) {
    if (tr && tid == 0) tr[kTrSplitArrived] = globaltimer_ns();
    const int ks_me = static_cast<int>(cluster_ctarank());
    Tile t;
    decode(p, static_cast<int>(blockIdx.x), t);
    const int c4n = p.kpad / 4;
    const int rs = (128 + p.S - 1) / p.S;
    const int row0 = ks_me * rs, nrows = min(128, row0 + rs) - row0;
    const int nitems = nrows > 0 ? nrows * c4n : 0;
    // four items per thread and pass, the loads of all four from up to four
    // partials in flight together (one round trip of distributed shared
    // memory per pass instead of one per item), summed in split order
    for (int i0 = tid; i0 < nitems; i0 += 4 * 128) {
      uint32_t off[4];
      bool valid[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int it = i0 + u * 128;
        valid[u] = it < nitems;
        const int c4 = valid[u] ? it / nrows : 0;
        const int row = valid[u] ? row0 + (it - c4 * nrows) : row0;
        off[u] = static_cast<uint32_t>(c4 * 128 + row);
      }
      float4 acc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int ks = 0; ks < p.S; ks += 4) {
        float4 v[4][4];
        load_partials_from(v, stage_u32, ks, p.S, off);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (ks + j < p.S)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              acc[u].x += v[j][u].x;
              acc[u].y += v[j][u].y;
              acc[u].z += v[j][u].z;
              acc[u].w += v[j][u].w;
            }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (!valid[u]) continue;
        const int c4 = static_cast<int>(off[u]) / 128, row = static_cast<int>(off[u]) - c4 * 128;
        const float f[4] = {acc[u].x, acc[u].y, acc[u].z, acc[u].w};
        store_row(p, t, row, 4 * c4, f);
      }
    }
    if (tr && tid == 0) tr[kTrSplitReduced] = globaltimer_ns();
  }
  static __device__ __forceinline__ void epilogue_drain(const Params&, EpiCtx&) {}
};
using GramPolicy = GramPolicyT<false, false>;
using GramLoPolicy = GramPolicyT<false, true>;
using GramAlsPolicy = GramPolicyT<true, false>;


// ================================================================ rfactor ====
// C^T = W_res . T'^T (d_out x B*k): A = W_res (K-major), B = T' (K-major).
// W_res is streamed from HBM once per n-tile column of C^T.
struct RFactorPolicy {
  // The solve's blocks (152 registers) run beside this GEMM's on the same SMs:
  // a register partition then holds two warps of each (2*152*32 + 2*104*32 =
  // 16384 registers), so the GEMM is held to 104.
  static constexpr int kMaxRegs = 104;
  static constexpr bool kBParts = true;  // split T: hi and lo parts per stage
  struct Params {
    GemmCommon c;
    CUtensorMap tmW;  // (d_in, d_out), box (64, 128)
    CUtensorMap tmT;  // (d_in, B*k),   box (64, bn)
    CUtensorMap tmC;  // (B*k, d_out),  box (64, 128), store
    CUtensorMap tmClo;  // same over the low parts (hilo)
    CUtensorMap tmTlo;  // the low parts of T (split T), like tmT
    int d_in, d_out, Bk, bn, n_tiles_n;
    int hilo;    // also store the low parts of Q^T
    int split_t;  // T arrives as hi and lo parts: a second B operand per stage
  };
  struct Tile {
    int m0, n0;
  };
  static constexpr uint32_t kEpiSmemBytes = kStoreBoxes * kStoreBoxBytes;

  static __device__ __forceinline__ void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmW);
    tma_prefetch_desc(&p.tmT);
    tma_prefetch_desc(&p.tmC);
    if (p.hilo) tma_prefetch_desc(&p.tmClo);
    if (p.split_t) tma_prefetch_desc(&p.tmTlo);
  }
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    t.m0 = (tile / p.n_tiles_n) * 128;
    t.n0 = (tile % p.n_tiles_n) * p.bn;
  }
  static __device__ __forceinline__ int kiters(const Params& p, const Tile&) {
    return ceil_div_dev(p.d_in, 64);
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar) {
    load_early(p, t, it, sa, sb, bar);
    load_late(p, t, it, sa, sb, bar);
  }
  // W_res is a loaded weight; T comes from the Gram stage, the grid before.
  static constexpr bool kEarly = true;
  static __device__ __forceinline__ void load_early(const Params& p, const Tile& t, int it,
                                                    uint32_t sa, uint32_t, uint32_t bar) {
    tma_load_2d(sa, &p.tmW, bar, it * 64, t.m0);
  }
  static __device__ __forceinline__ void load_late(const Params& p, const Tile& t, int it,
                                                   uint32_t, uint32_t sb, uint32_t bar) {
    tma_load_2d(sb, &p.tmT, bar, it * 64, t.n0);
    if (p.split_t) tma_load_2d(sb + static_cast<uint32_t>(p.bn) * 128u, &p.tmTlo, bar, it * 64, t.n0);
  }
  static __device__ __forceinline__ int ksteps(const Params& p, const Tile&, int it) {
    return min(4, ceil_div_dev(p.d_in - it * 64, 16));
  }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    return kmajor_desc(a, ks);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params&, uint32_t b, int ks) {
    return kmajor_desc(b, ks);
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    for (int bx = 0; bx < p.bn / 64; ++bx) {
      store_box_bf16(tacc, bx * 64, &p.tmC, t.n0 + bx * 64, t.m0, e);
      if (p.hilo) store_box_bf16<true>(tacc, bx * 64, &p.tmClo, t.n0 + bx * 64, t.m0, e);
    }
  }
  static __device__ __forceinline__ bool cluster_finish(const Params&) { return false; }
  static __device__ __forceinline__ void finish(const Params&, int, uint32_t, unsigned long long*) {}
  static __device__ __forceinline__ void epilogue_drain(const Params&, EpiCtx& e) { store_drain(e); }
};

// ==================================================================== out ====
// Y = Z U^T + sum over the instances b the m-tile touches of mask_b(L) C_b,
// accumulated in one TMEM tile: K-segments [Z | L_b_lo | ... | L_b_hi] against
// [U ; C_b_lo ; ... ; C_b_hi]. mask_b(L) is L's rows of instance b and zero
// elsewhere, produced by TMA's out-of-bounds fill on the 3-D view of L.
// The bf16 result goes out through swizzled shared-memory boxes and TMA
// stores; two boxes rotate, so one store drains while the next box is
// written (more boxes would cost a pipeline stage).
struct OutParams {
    GemmCommon c;
    CUtensorMap tmZ;  // (r, N),        box (64, 128)
    CUtensorMap tmU;  // (r, d_out),    box (64, bn)
    CUtensorMap tmL;  // (k, T, B),     box (64, 128, 1)
    CUtensorMap tmC;  // (B*k, d_out),  box (64, bn)
    CUtensorMap tmY;  // (d_out, N),    box (64, 128), store
    CUtensorMap tmLlo, tmClo;  // the low parts of L~ and Q^T (hilo)
    int N, r, k, T, B, bn, n_tiles_n, nkz, nkl;
    const __nv_bfloat16* bias;  // d_out, added in the epilogue, or nullptr
    int d_out;
    int hilo;  // correction as hi L~ . hi Q + hi L~ . lo Q + lo L~ . hi Q
    // Block-diagonal static part (zb_w > 0; a Monarch factor, [DyRA] App. B):
    // output columns come in zb_n blocks of zb_w, and block c is the product
    // of Z's columns c*zb_k .. + zb_k with block c of U, read through the 3-D
    // view tmU (zb_k, zb_w, zb_n), box (64, rows, 1), whose out-of-bounds fill
    // zeroes the tile's rows outside the block. nkz is then the K-steps of one
    // block. zb_w == 0: the dense Z U^T (K = r).
    int zb_w, zb_k, zb_n;
    // 1 (k <= 32): the correction's boxes are 32 columns wide (64-byte
    // swizzle), half the bytes of a 64-wide box, of which k <= 32 columns
    // would be used; its stages then hold 64-byte rows
    int narrow;
};

// kExt compiles in the compensated correction (hilo) and the block-diagonal
// static part (zb_w > 0), kBias the bias. The plain layer runs
// OutPolicyT<false, false>, which ignores those fields.
template <bool kExt, bool kBias>
struct OutPolicyT {
  using Params = OutParams;
  // The static part's blocks that the tile's columns n0 .. n0 + bn - 1 touch.
  static __device__ __forceinline__ void static_blocks(const Params& p, int n0, int& lo,
                                                       int& nseg) {
    if (kExt && p.zb_w > 0) {
      lo = n0 / p.zb_w;
      nseg = min(p.zb_n - 1, (n0 + p.bn - 1) / p.zb_w) - lo + 1;
    } else {
      lo = 0;
      nseg = 1;
    }
  }
  static __device__ __forceinline__ int static_iters(const Params& p, int z_nseg) {
    return kExt && p.zb_w > 0 ? z_nseg * p.nkz : p.nkz;
  }
  static __device__ __forceinline__ int static_ksteps(const Params& p, int it) {
    if (kExt && p.zb_w > 0) return min(4, ceil_div_dev(p.zb_k - (it % p.nkz) * 64, 16));
    return min(4, ceil_div_dev(p.r - it * 64, 16));
  }
  // K-step j of the correction: instance segment, sub-product (0 hi.hi,
  // 1 hi.lo, 2 lo.hi) and 64-wide chunk of k.
  static __device__ __forceinline__ void correction_step(const Params& p, int j, int& seg,
                                                         int& sub, int& ch) {
    const int per = p.nkl * (kExt && p.hilo ? 3 : 1);
    seg = j / per;
    const int jj = j - seg * per;
    sub = jj / p.nkl;
    ch = jj - sub * p.nkl;
  }
  struct Tile {
    int m0, n0, b_lo, nseg, z_lo, z_nseg, ns;  // ns: the static part's K-steps
  };
  static constexpr uint32_t kEpiSmemBytes = kStoreBoxes * kStoreBoxBytes;

  static __device__ __forceinline__ void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmZ);
    tma_prefetch_desc(&p.tmU);
    if (p.nkl > 0) {
      tma_prefetch_desc(&p.tmL);
      tma_prefetch_desc(&p.tmC);
      if (kExt && p.hilo) {
        tma_prefetch_desc(&p.tmLlo);
        tma_prefetch_desc(&p.tmClo);
      }
    }
    tma_prefetch_desc(&p.tmY);
  }
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    t.m0 = (tile / p.n_tiles_n) * 128;
    t.n0 = (tile % p.n_tiles_n) * p.bn;
    if (p.nkl > 0) {
      t.b_lo = t.m0 / p.T;
      const int b_hi = min(p.B - 1, (t.m0 + 127) / p.T);
      t.nseg = b_hi - t.b_lo + 1;
    } else {
      t.b_lo = 0;
      t.nseg = 0;
    }
    static_blocks(p, t.n0, t.z_lo, t.z_nseg);
    t.ns = static_iters(p, t.z_nseg);
  }
  static __device__ __forceinline__ int kiters(const Params& p, const Tile& t) {
    return t.ns + t.nseg * p.nkl * (kExt && p.hilo ? 3 : 1);
  }
  // With Params::early (set only where the grid chain guarantees it: the
  // rank-k GEMM before the solve triggers its dependents only after its own
  // wait, so Z of the projection is complete before this grid launches) the
  // static stages (Z and U) are loaded before the dependency wait and their
  // MMAs may run before it ends; the correction's operands come after it.
  static constexpr bool kEarly = true;
  static __device__ __forceinline__ void load_early(const Params& p, const Tile& t, int it,
                                                    uint32_t sa, uint32_t sb, uint32_t bar) {
    if (it < t.ns) load(p, t, it, sa, sb, bar);
  }
  static __device__ __forceinline__ void load_late(const Params& p, const Tile& t, int it,
                                                   uint32_t sa, uint32_t sb, uint32_t bar) {
    if (it >= t.ns) load(p, t, it, sa, sb, bar);
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar) {
    const int ns = t.ns;
    if (it < ns) {
      if (kExt && p.zb_w > 0) {
        const int seg = it / p.nkz, kk = it - seg * p.nkz, blk = t.z_lo + seg;
        tma_load_2d(sa, &p.tmZ, bar, blk * p.zb_k + kk * 64, t.m0);
        tma_load_3d(sb, &p.tmU, bar, kk * 64, t.n0 - blk * p.zb_w, blk);
      } else {
        tma_load_2d(sa, &p.tmZ, bar, it * 64, t.m0);
        tma_load_2d(sb, &p.tmU, bar, it * 64, t.n0);
      }
    } else {
      int seg, sub, ch;
      correction_step(p, it - ns, seg, sub, ch);
      const int b = t.b_lo + seg;
      tma_load_3d(sa, kExt && sub == 2 ? &p.tmLlo : &p.tmL, bar, ch * 64, t.m0 - b * p.T, b);
      tma_load_2d(sb, kExt && sub == 1 ? &p.tmClo : &p.tmC, bar, b * p.k + ch * 64, t.n0);
    }
  }
  static __device__ __forceinline__ int ksteps(const Params& p, const Tile& t, int it) {
    if (it < t.ns) return static_ksteps(p, it);
    const int ch = (it - t.ns) % p.nkl;
    return min(4, ceil_div_dev(p.k - ch * 64, 16));
  }
  // narrow correction stages: half the bytes, K-major rows of 64 bytes
  // (8-row atoms 512 bytes apart); the k-th group of 16 columns is 32 bytes
  // further into each row, as in the 128-byte layout
  static constexpr bool kStageLayouts = true;
  static __device__ __forceinline__ bool narrow_stage(const Params& p, const Tile& t, int it) {
    return p.narrow && it >= t.ns;
  }
  static __device__ __forceinline__ uint32_t stage_tx(const Params& p, const Tile& t, int it) {
    const uint32_t full = p.c.a_stage_bytes + p.c.b_stage_bytes;
    return narrow_stage(p, t, it) ? full / 2 : full;
  }
  static __device__ __forceinline__ uint64_t stage_adesc(const Params& p, const Tile& t, int it,
                                                         uint32_t a) {
    return narrow_stage(p, t, it) ? smem_desc(a, 16u, 512u, kLayoutSw64) : kmajor_desc(a, 0);
  }
  static __device__ __forceinline__ uint64_t stage_bdesc(const Params& p, const Tile& t, int it,
                                                         uint32_t b) {
    return narrow_stage(p, t, it) ? smem_desc(b, 16u, 512u, kLayoutSw64) : kmajor_desc(b, 0);
  }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    return kmajor_desc(a, ks);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params&, uint32_t b, int ks) {
    return kmajor_desc(b, ks);
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    if (kBias && p.bias != nullptr) {
      for (int bx = 0; bx < p.bn / 64; ++bx)
        store_box_bf16<false, true>(tacc, bx * 64, &p.tmY, t.n0 + bx * 64, t.m0, e, p.bias,
                                    p.d_out);
    } else {
      for (int bx = 0; bx < p.bn / 64; ++bx)
        store_box_bf16(tacc, bx * 64, &p.tmY, t.n0 + bx * 64, t.m0, e);
    }
  }
  static __device__ __forceinline__ bool cluster_finish(const Params&) { return false; }
  static __device__ __forceinline__ void finish(const Params&, int, uint32_t, unsigned long long*) {}
  static __device__ __forceinline__ void epilogue_drain(const Params&, EpiCtx& e) { store_drain(e); }
};

// ============================================================= x . rw^T ====
// The left update of a further ALS iteration ([DyRA] Eq. 4) needs, per
// instance b, P2_b = X_b (R_b W_res)^T (T x k). Tile: 128 rows of X (through
// the (d_in, T, B) view, so each instance segment of a tile that straddles
// instances is masked by the copy's out-of-bounds fill, as in the output
// stage) times the k x d_in block of R W_res of that instance (K-major B
// operand, rows b*k ..), K = d_in per segment. The accumulator's first k
// columns leave as bf16 rows of P2 (N x k) through 16-byte stores.
struct XRwPolicy {
  struct Params {
    GemmCommon c;
    CUtensorMap tmX;   // (d_in, T, B), box (64, 128, 1)
    CUtensorMap tmRW;  // (d_in, B*k),  box (64, kpad)
    __nv_bfloat16* P2;  // N x k
    int N, d_in, k, kpad, T, B, nkd;
  };
  struct Tile {
    int m0, b_lo, nseg;
  };
  static constexpr uint32_t kEpiSmemBytes = 0;

  static __device__ __forceinline__ void prefetch(const Params& p) {
    tma_prefetch_desc(&p.tmX);
    tma_prefetch_desc(&p.tmRW);
  }
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    t.m0 = tile * 128;
    t.b_lo = t.m0 / p.T;
    const int b_hi = min(p.B - 1, (t.m0 + 127) / p.T);
    t.nseg = b_hi - t.b_lo + 1;
  }
  static __device__ __forceinline__ int kiters(const Params& p, const Tile& t) {
    return t.nseg * p.nkd;
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar) {
    const int seg = it / p.nkd;
    const int ch = it - seg * p.nkd;
    const int b = t.b_lo + seg;
    tma_load_3d(sa, &p.tmX, bar, ch * 64, t.m0 - b * p.T, b);
    tma_load_2d(sb, &p.tmRW, bar, ch * 64, b * p.k);
  }
  static __device__ __forceinline__ int ksteps(const Params& p, const Tile&, int it) {
    const int ch = it % p.nkd;
    return min(4, ceil_div_dev(p.d_in - ch * 64, 16));
  }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    return kmajor_desc(a, ks);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params&, uint32_t b, int ks) {
    return kmajor_desc(b, ks);
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    const int row = t.m0 + e.row;
    for (int cc = 0; cc < p.kpad; cc += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + cc, v);
      tmem_ld_wait();
      if (row >= p.N) continue;
      __nv_bfloat16* dst = p.P2 + static_cast<size_t>(row) * p.k + cc;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        if (cc + 8 * c8 >= p.k) break;  // k is a multiple of 8
        if (!in_bounds(p.c.status, (dst - p.P2) + 8 * c8, 8, static_cast<size_t>(p.N) * p.k))
          break;
        uint4 q;
        q.x = pack_bf16x2(f32(v[8 * c8 + 0]), f32(v[8 * c8 + 1]));
        q.y = pack_bf16x2(f32(v[8 * c8 + 2]), f32(v[8 * c8 + 3]));
        q.z = pack_bf16x2(f32(v[8 * c8 + 4]), f32(v[8 * c8 + 5]));
        q.w = pack_bf16x2(f32(v[8 * c8 + 6]), f32(v[8 * c8 + 7]));
        *reinterpret_cast<uint4*>(dst + 8 * c8) = q;
      }
    }
  }
  static __device__ __forceinline__ bool cluster_finish(const Params&) { return false; }
  static __device__ __forceinline__ void finish(const Params&, int, uint32_t, unsigned long long*) {}
  static __device__ __forceinline__ void epilogue_drain(const Params&, EpiCtx&) {}
};

// ============================================================ proj, pairs ====
// C^T = W_res T'^T on CTA pairs: tile 256 x bn, CTA r loads rows m0 + 128 r
// of W_res and rows n0 + (bn/2) r of T' and stores its 128 rows of C^T.
struct RFactorPairPolicy {
  using Params = RFactorPolicy::Params;  // tmT box is (64, bn/2) here
  static constexpr int kMaxRegs = RFactorPolicy::kMaxRegs;
  static constexpr bool kBParts = RFactorPolicy::kBParts;
  using Tile = RFactorPolicy::Tile;
  static constexpr uint32_t kEpiSmemBytes = RFactorPolicy::kEpiSmemBytes;
  static __device__ __forceinline__ void prefetch(const Params& p) { RFactorPolicy::prefetch(p); }
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    t.m0 = (tile / p.n_tiles_n) * 256;
    t.n0 = (tile % p.n_tiles_n) * p.bn;
  }
  static __device__ __forceinline__ int kiters(const Params& p, const Tile& t) {
    return RFactorPolicy::kiters(p, t);
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar, uint32_t rank) {
    load_early(p, t, it, sa, sb, bar, rank);
    load_late(p, t, it, sa, sb, bar, rank);
  }
  static constexpr bool kEarly = true;  // as RFactorPolicy: W_res early, T late
  static __device__ __forceinline__ void load_early(const Params& p, const Tile& t, int it,
                                                    uint32_t sa, uint32_t, uint32_t bar,
                                                    uint32_t rank) {
    tma_load_2d_pair(sa, &p.tmW, bar, it * 64, t.m0 + 128 * static_cast<int>(rank));
  }
  static __device__ __forceinline__ void load_late(const Params& p, const Tile& t, int it,
                                                   uint32_t, uint32_t sb, uint32_t bar,
                                                   uint32_t rank) {
    tma_load_2d_pair(sb, &p.tmT, bar, it * 64, t.n0 + (p.bn / 2) * static_cast<int>(rank));
    if (p.split_t)
      tma_load_2d_pair(sb + static_cast<uint32_t>(p.bn / 2) * 128u, &p.tmTlo, bar, it * 64,
                       t.n0 + (p.bn / 2) * static_cast<int>(rank));
  }
  static __device__ __forceinline__ int ksteps(const Params& p, const Tile& t, int it) {
    return RFactorPolicy::ksteps(p, t, it);
  }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    return kmajor_desc(a, ks);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params&, uint32_t b, int ks) {
    return kmajor_desc(b, ks);
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    Tile h{t.m0 + 128 * e.rank, t.n0};
    RFactorPolicy::epilogue(p, h, tacc, e);
  }
  static __device__ __forceinline__ void epilogue_drain(const Params& p, EpiCtx& e) {
    RFactorPolicy::epilogue_drain(p, e);
  }
};

// [Z | L] = X [V | P] on CTA pairs: tile 256 x bn, CTA r loads rows
// m0 + 128 r of X and rows n0 + (bn/2) r of [V | P]^T and stores its 128 rows.
struct ProjPairPolicy {
  using Params = ProjPolicy::Params;  // tmW box is (64, bn/2) here
  using Tile = ProjPolicy::Tile;
  static constexpr uint32_t kEpiSmemBytes = ProjPolicy::kEpiSmemBytes;
  static __device__ __forceinline__ void prefetch(const Params& p) { ProjPolicy::prefetch(p); }
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    t.m0 = (tile / p.n_tiles_n) * 256;
    t.n0 = (tile % p.n_tiles_n) * p.bn;
    t.ks = 0;
    t.base = tile;
  }
  static __device__ __forceinline__ int kiters(const Params& p, const Tile& t) {
    return ProjPolicy::kiters(p, t);
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar, uint32_t rank) {
    load_early(p, t, it, sa, sb, bar, rank);
    load_late(p, t, it, sa, sb, bar, rank);
  }
  static constexpr bool kEarly = true;  // as ProjPolicy: [V | P]^T early, X late
  static __device__ __forceinline__ void load_early(const Params& p, const Tile& t, int it,
                                                    uint32_t, uint32_t sb, uint32_t bar,
                                                    uint32_t rank) {
    tma_load_2d_pair(sb, &p.tmW, bar, it * 64, t.n0 + (p.bn / 2) * static_cast<int>(rank));
  }
  static __device__ __forceinline__ void load_late(const Params& p, const Tile& t, int it,
                                                   uint32_t sa, uint32_t, uint32_t bar,
                                                   uint32_t rank) {
    tma_load_2d_pair(sa, &p.tmX, bar, it * 64, t.m0 + 128 * static_cast<int>(rank));
  }
  static __device__ __forceinline__ int ksteps(const Params& p, const Tile& t, int it) {
    return ProjPolicy::ksteps(p, t, it);
  }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    return kmajor_desc(a, ks);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params&, uint32_t b, int ks) {
    return kmajor_desc(b, ks);
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    Tile h{t.m0 + 128 * e.rank, t.n0, 0, t.base};
    ProjPolicy::epilogue(p, h, tacc, e);
  }
  static __device__ __forceinline__ void epilogue_drain(const Params& p, EpiCtx& e) {
    ProjPolicy::epilogue_drain(p, e);
  }
};

// =============================================================== out, pairs ====
// The output stage on CTA pairs: tile 256 x bn, CTA r of the pair owns rows
// m0 + 128 r .. +127 of A and of Y, and rows n0 + (bn/2) r .. + bn/2 - 1 of
// the B operand ([U ; C_b]); the epilogue is OutPolicyT's for its 128 rows.
template <bool kExt, bool kBias>
struct OutPairPolicyT {
  using Single = OutPolicyT<kExt, kBias>;
  using Params = OutParams;  // tmU / tmC boxes are (64, bn/2) here
  struct Tile {
    int m0, n0, b_lo, nseg, z_lo, z_nseg, ns;
  };
  static constexpr uint32_t kEpiSmemBytes = Single::kEpiSmemBytes;

  static __device__ __forceinline__ void prefetch(const Params& p) { Single::prefetch(p); }
  static __device__ __forceinline__ void decode(const Params& p, int tile, Tile& t) {
    t.m0 = (tile / p.n_tiles_n) * 256;
    t.n0 = (tile % p.n_tiles_n) * p.bn;
    if (p.nkl > 0) {
      t.b_lo = t.m0 / p.T;
      const int b_hi = min(p.B - 1, (t.m0 + 255) / p.T);
      t.nseg = b_hi - t.b_lo + 1;
    } else {
      t.b_lo = 0;
      t.nseg = 0;
    }
    Single::static_blocks(p, t.n0, t.z_lo, t.z_nseg);
    t.ns = Single::static_iters(p, t.z_nseg);
  }
  static __device__ __forceinline__ int kiters(const Params& p, const Tile& t) {
    return t.ns + t.nseg * p.nkl * (kExt && p.hilo ? 3 : 1);
  }
  static constexpr bool kEarly = true;  // as OutPolicyT: static stages early
  static __device__ __forceinline__ void load_early(const Params& p, const Tile& t, int it,
                                                    uint32_t sa, uint32_t sb, uint32_t bar,
                                                    uint32_t rank) {
    if (it < t.ns) load(p, t, it, sa, sb, bar, rank);
  }
  static __device__ __forceinline__ void load_late(const Params& p, const Tile& t, int it,
                                                   uint32_t sa, uint32_t sb, uint32_t bar,
                                                   uint32_t rank) {
    if (it >= t.ns) load(p, t, it, sa, sb, bar, rank);
  }
  static __device__ __forceinline__ void load(const Params& p, const Tile& t, int it, uint32_t sa,
                                              uint32_t sb, uint32_t bar, uint32_t rank) {
    const int ma = t.m0 + 128 * static_cast<int>(rank);
    const int nb = t.n0 + (p.bn / 2) * static_cast<int>(rank);
    const int ns = t.ns;
    if (it < ns) {
      if (kExt && p.zb_w > 0) {
        const int seg = it / p.nkz, kk = it - seg * p.nkz, blk = t.z_lo + seg;
        tma_load_2d_pair(sa, &p.tmZ, bar, blk * p.zb_k + kk * 64, ma);
        tma_load_3d_pair(sb, &p.tmU, bar, kk * 64, nb - blk * p.zb_w, blk);
      } else {
        tma_load_2d_pair(sa, &p.tmZ, bar, it * 64, ma);
        tma_load_2d_pair(sb, &p.tmU, bar, it * 64, nb);
      }
    } else {
      int seg, sub, ch;
      Single::correction_step(p, it - ns, seg, sub, ch);
      const int b = t.b_lo + seg;
      tma_load_3d_pair(sa, kExt && sub == 2 ? &p.tmLlo : &p.tmL, bar, ch * 64, ma - b * p.T, b);
      tma_load_2d_pair(sb, kExt && sub == 1 ? &p.tmClo : &p.tmC, bar, b * p.k + ch * 64, nb);
    }
  }
  static __device__ __forceinline__ int ksteps(const Params& p, const Tile& t, int it) {
    if (it < t.ns) return Single::static_ksteps(p, it);
    const int ch = (it - t.ns) % p.nkl;
    return min(4, ceil_div_dev(p.k - ch * 64, 16));
  }
  static constexpr bool kStageLayouts = true;  // as Single: narrow correction stages
  static __device__ __forceinline__ uint32_t stage_tx(const Params& p, const Tile& t, int it) {
    const uint32_t full = p.c.a_stage_bytes + p.c.b_stage_bytes;
    return p.narrow && it >= t.ns ? full / 2 : full;
  }
  static __device__ __forceinline__ uint64_t stage_adesc(const Params& p, const Tile& t, int it,
                                                         uint32_t a) {
    return p.narrow && it >= t.ns ? smem_desc(a, 16u, 512u, kLayoutSw64) : kmajor_desc(a, 0);
  }
  static __device__ __forceinline__ uint64_t stage_bdesc(const Params& p, const Tile& t, int it,
                                                         uint32_t b) {
    return p.narrow && it >= t.ns ? smem_desc(b, 16u, 512u, kLayoutSw64) : kmajor_desc(b, 0);
  }
  static __device__ __forceinline__ uint64_t adesc(const Params&, uint32_t a, int ks) {
    return kmajor_desc(a, ks);
  }
  static __device__ __forceinline__ uint64_t bdesc(const Params&, uint32_t b, int ks) {
    return kmajor_desc(b, ks);
  }
  static __device__ __forceinline__ void epilogue(const Params& p, const Tile& t, uint32_t tacc,
                                                  EpiCtx& e) {
    typename Single::Tile h;
    h.m0 = t.m0 + 128 * e.rank;
    h.n0 = t.n0;
    h.b_lo = t.b_lo;
    h.nseg = t.nseg;
    h.z_lo = t.z_lo;
    h.z_nseg = t.z_nseg;
    h.ns = t.ns;
    Single::epilogue(p, h, tacc, e);
  }
  static __device__ __forceinline__ void epilogue_drain(const Params& p, EpiCtx& e) {
    Single::epilogue_drain(p, e);
  }
};

// ============================================================= host side ====

namespace {

inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

uint32_t pow2_at_least(uint32_t x) {
  uint32_t v = 32;
  while (v < x) v <<= 1;
  return v;
}

// Fill the shared part of the launch parameters; returns dynamic smem bytes
// or 0 if the tile shape does not fit.
template <class Pol>
uint32_t setup_common(GemmCommon& c, int num_tiles, uint32_t a_bytes, uint32_t b_bytes,
                      int mma_n, bool a_mn, bool b_mn, int* status, const DeviceInfo& dev,
                      int smem_cap = 0) {
  c.num_tiles = num_tiles;
  c.defer_wait = 0;
  c.trigger_after_wait = 0;
  c.b_parts = 1;
  c.b_part_desc = 0;
  c.wait_ns = sm100::kWaitLimitNs;
  c.early = 0;
  c.a_stage_bytes = a_bytes;
  c.b_stage_bytes = b_bytes;
  c.acc_cols = static_cast<uint32_t>((mma_n + 31) / 32 * 32);
  c.tmem_cols = pow2_at_least(2 * c.acc_cols);
  if (c.tmem_cols > 512) return 0;
  c.idesc = idesc_bf16(128, mma_n, a_mn, b_mn);
  c.status = status;
  c.trace = nullptr;
  const uint32_t fixed = gemm_smem_bytes(0, a_bytes, b_bytes, Pol::kEpiSmemBytes);
  const int full = (dev.max_smem_optin - static_cast<int>(fixed)) / static_cast<int>(a_bytes + b_bytes);
  int stages = full;
  if (smem_cap > 0) {
    // a cap that would leave fewer than 3 stages is not worth its room
    const int capped = (std::min(smem_cap, dev.max_smem_optin) - static_cast<int>(fixed)) /
                       static_cast<int>(a_bytes + b_bytes);
    if (capped >= 3) stages = capped;
  }
  stages = std::min(stages, kMaxStages);
  if (stages < 2) return 0;
  c.stages = stages;
  return gemm_smem_bytes(stages, a_bytes, b_bytes, Pol::kEpiSmemBytes);
}

template <class Pol>
int launch_gemm(const typename Pol::Params& p, uint32_t smem, const DeviceInfo& dev,
                cudaStream_t s, bool pdl, int cluster = 1) {
  if (p.c.num_tiles <= 0) return 0;
  auto kfn = umma_gemm_kernel<Pol>;
  static KernelSetup setup;
  const int d = dev.device;
  if (d < 0 || d >= kMaxDevices) return -1;
  if (smem > setup.smem[d].load()) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(kfn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
            cudaSuccess)
      return -1;
    setup.smem[d].store(smem);
  }
  cudaLaunchConfig_t cfg = {};
  // with clusters every CTA takes exactly one tile (the grid is the tile count)
  cfg.gridDim = dim3(static_cast<unsigned>(
      cluster > 1 ? p.c.num_tiles : std::min(p.c.num_tiles, dev.sm_count)));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster > 1) {
    if (p.c.num_tiles % cluster != 0) return -1;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(na);
  return cudaLaunchKernelEx(&cfg, kfn, p) == cudaSuccess ? 0 : -1;
}

template <class Pol>
int launch_gemm_pair(const typename Pol::Params& p, uint32_t smem, const DeviceInfo& dev,
                     cudaStream_t s, bool pdl) {
  if (p.c.num_tiles <= 0) return 0;
  auto kfn = umma_gemm_pair_kernel<Pol>;
  static KernelSetup setup;  // occupancy: resident pairs at the configured size
  const int d = dev.device;
  if (d < 0 || d >= kMaxDevices) return -1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  if (smem > setup.smem[d].load() || setup.occupancy[d].load() < 1) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(kfn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
            cudaSuccess)
      return -1;
    cfg.gridDim = dim3(2 * (dev.sm_count / 2));
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kfn, &cfg) != cudaSuccess || clusters < 1) {
      cudaGetLastError();
      clusters = dev.sm_count / 2;
    }
    setup.occupancy[d].store(clusters);
    if (smem > setup.smem[d].load()) setup.smem[d].store(smem);
  }
  const int max_pairs = setup.occupancy[d].load();
  cfg.gridDim = dim3(static_cast<unsigned>(2 * std::min(p.c.num_tiles, max_pairs)));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kfn, p) == cudaSuccess ? 0 : -1;
}

// Column tile for a K-major B operand of n columns: at most 256 wide, a
// multiple of 32, chosen so the tiles split n evenly.
int pick_bn(int n) {
  const int tiles = ceil_div(n, 256);
  int bn = ceil_div(ceil_div(n, tiles), 32) * 32;
  return std::min(bn, 256);
}

}  // namespace

ProjShape proj_shape(int64_t N, int d_in, int r, int k_eff, bool use_pairs, int sm_count,
                     int pair_min_tiles, int force_bn) {
  ProjShape ps;
  const int n_cols = r + k_eff;
  ps.tma_store = (r % 64 == 0 && k_eff <= 64) ? 1 : 0;
  // Column tile and CTA pairs: the stage is bound by the bytes each CTA
  // streams per k-step (128 rows of X, plus bn / 2 rows of [V | P]^T on a
  // pair or bn rows alone) times the rounds of tiles per SM. Pick the
  // cheapest of bn = 128, 192, 256 (whole 64-column store boxes) and the
  // width that splits the columns evenly over the fewest tiles (a multiple
  // of 16; e.g. 2 x 144 for 288 columns instead of 2 x 192), whose stores
  // then go out as 16-byte row pieces.
  const int pair_min = pair_min_tiles > 0 ? pair_min_tiles : sm_count / 4;
  const int exact =
      std::min(256, ceil_div(ceil_div(n_cols, std::max(1, ceil_div(n_cols, 256))), 16) * 16);
  int64_t best = -1;
  for (int bn : {192, 256, 128, exact}) {
    if (force_bn > 0 && bn != force_bn) continue;
    if (bn == exact && force_bn != exact && (exact % 64 == 0 || exact < 16)) continue;
    const int nt = ceil_div(n_cols, bn);
    for (int pairs = 1; pairs >= 0; --pairs) {
      if (pairs && !use_pairs) continue;
      const int64_t tiles = (pairs ? ceil_div(N, 256) : ceil_div(N, 128)) * nt;
      if (pairs && tiles < pair_min) continue;
      const int64_t slots = pairs ? sm_count / 2 : sm_count;
      const int64_t cost = (tiles + slots - 1) / slots * (128 + (pairs ? bn / 2 : bn));
      if (best < 0 || cost < best) {
        best = cost;
        ps.bn = bn;
        ps.n_tiles_n = nt;
        ps.pairs = pairs != 0;
        ps.tiles = static_cast<int>(tiles);
      }
    }
  }
  if (ps.bn % 64 != 0) ps.tma_store = 0;
  ps.ksplit = 1;
  const int kit = ceil_div(d_in, 64);
  ps.kper = kit;
  if (!ps.pairs && ps.tiles * 2 <= sm_count && kit >= 8) {
    // Split-K: narrower column tiles first (more tiles, and half the fp32
    // partial each CTA sums over the cluster), then up to 8 splits per tile
    // (portable cluster size).
    if (ps.bn > 128 || ps.bn % 32 != 0) {  // whole 32-column TMEM loads into the partial
      ps.bn = 128;
      ps.n_tiles_n = ceil_div(n_cols, ps.bn);
      ps.tiles = static_cast<int>(ceil_div(N, 128)) * ps.n_tiles_n;
      ps.tma_store = (r % 64 == 0 && k_eff <= 64) ? 1 : 0;
    }
    const int want = std::min(sm_count / ps.tiles, std::min(kit / 4, 8));
    if (want > 1) {
      ps.kper = ceil_div(kit, want);
      ps.ksplit = ceil_div(kit, ps.kper);
    }
  }
  return ps;
}

int factor_record_floats(int k) {
  if (k <= 0 || k > 64) return 0;
  return k <= 32 ? ldl_record_floats<32>() : ldl_record_floats<64>();
}

void gram_split(int64_t T, int64_t B, int d_in, int k, int sm_count, int* splits,
                int* split_rows) {
  // Split each instance's rows (whole 64-row blocks) to balance the tiles
  // over the SMs. A tile costs about 2 us of pipeline fill and epilogue plus
  // 0.3 us per pipelined 64-row block, and a split tile 3 us more for the
  // reduction of the partials over distributed shared memory (per-CTA
  // timelines of the Gram stage); rounds of tiles per SM multiply it.
  const int64_t blocks = (T + 63) / 64;
  const int64_t mtiles = (d_in + 127) / 128 + (k + 127) / 128;
  const int64_t per_split_tiles = std::max<int64_t>(1, B * mtiles);
  int64_t best_s = 1;
  double best = 0.0;
  for (int64_t sp = 1; sp <= std::min<int64_t>(8, blocks); ++sp) {
    const int64_t per = (blocks + sp - 1) / sp;
    const int64_t used = (blocks + per - 1) / per;  // splits actually made
    if (used != sp) continue;
    const int64_t rounds = (per_split_tiles * sp + sm_count - 1) / sm_count;
    const double tile_us = 2.0 + 0.3 * static_cast<double>(per) + (sp > 1 ? 3.0 : 0.0);
    const double cost = static_cast<double>(rounds) * tile_us;
    if (sp == 1 || cost < best) {
      best = cost;
      best_s = sp;
    }
  }
  const int64_t per = (blocks + best_s - 1) / best_s;
  *split_rows = static_cast<int>(per * 64);
  *splits = static_cast<int>((blocks + per - 1) / per);
}

namespace {

// One Gram stage (GramPolicy) over a pair of 3-D row views: X (d_in, rows,
// instances of X) and L (k, rows, B), strides in bytes. The one-step forward
// runs it over (X_b, L_b); the L update of further ALS iterations over
// (W_res, R_b^T), with rows = d_out.
struct GramStage {
  const void* X;
  uint64_t xd[3], xs[2];
  int x_inst_fixed;
  const void* L;
  uint64_t ld[3], ls[2];
  int d_in, k, rows, B, S, Ts;
  __nv_bfloat16* Tb;
  __nv_bfloat16* Tlo;
  float* G;
  float* TGf;
  unsigned long long* trace;
  unsigned long long wait_ns;
};

template <class Pol>
int launch_gram_stage_as(const GramStage& g, int* status, const DeviceInfo& dev, cudaStream_t s,
                         bool pdl) {
  typename Pol::Params p;
  p.d_in = g.d_in;
  p.k = g.k;
  p.kpad = g.k <= 32 ? 32 : ceil_div(g.k, 64) * 64;
  p.w = std::min(p.kpad, 64);
  p.nbox_b = p.kpad / p.w;
  p.T = g.rows;
  p.B = g.B;
  p.S = g.S;
  p.Ts = g.Ts;
  p.mtx = ceil_div(g.d_in, 128);
  p.mt_total = p.mtx + ceil_div(g.k, 128);
  p.x_inst_fixed = g.x_inst_fixed;
  p.Tb = g.Tb;
  p.Tlo = g.Tlo;
  p.G = g.G;
  p.TGf = g.TGf;
  p.b_layout = p.w == 64 ? kLayoutSw128 : kLayoutSw64;  // w is 32 or 64
  uint32_t bx[3] = {64, 64, 1};
  if (!encode_tmap_bf16(&p.tmX, g.X, 3, g.xd, g.xs, bx, 128)) return -2;
  if (!encode_tmap_bf16(&p.tmLa, g.L, 3, g.ld, g.ls, bx, 128)) return -2;
  uint32_t bl[3] = {static_cast<uint32_t>(p.w), 64, 1};
  if (!encode_tmap_bf16(&p.tmLb, g.L, 3, g.ld, g.ls, bl, p.w * 2)) return -2;
  const int tiles = p.mt_total * p.B * p.S;
  const uint32_t smem =
      setup_common<Pol>(p.c, tiles, 128 * 128, static_cast<uint32_t>(p.kpad) * 128,
                               p.kpad, true, true, status, dev);
  if (!smem) return -3;
  // split rows keep a 128 x kpad fp32 partial in the operand stages
  if (p.S > 1 && static_cast<size_t>(p.c.stages) * (p.c.a_stage_bytes + p.c.b_stage_bytes) <
                     static_cast<size_t>(128) * p.kpad * 4)
    return -3;
  p.c.trace = g.trace;
  if (g.wait_ns) p.c.wait_ns = g.wait_ns;
  return launch_gemm<Pol>(p, smem, dev, s, pdl, p.S) ? -1 : 0;
}

int launch_gram_stage(const GramStage& g, int* status, const DeviceInfo& dev, cudaStream_t s,
                      bool pdl) {
  if (g.TGf != nullptr || g.x_inst_fixed) {
    if (g.Tlo != nullptr) return -3;  // no split T in the fp32 layout
    return launch_gram_stage_as<GramAlsPolicy>(g, status, dev, s, pdl);
  }
  return g.Tlo != nullptr ? launch_gram_stage_as<GramLoPolicy>(g, status, dev, s, pdl)
                          : launch_gram_stage_as<GramPolicy>(g, status, dev, s, pdl);
}

// The Gram stage of the layer: L_b^T [X_b | L_b] per instance, L = a.L.
GramStage layer_gram(const Bf16Forward& a) {
  GramStage g = {};
  g.X = a.X;
  g.xd[0] = static_cast<uint64_t>(a.d_in);
  g.xd[1] = static_cast<uint64_t>(a.T);
  g.xd[2] = static_cast<uint64_t>(a.B);
  g.xs[0] = static_cast<uint64_t>(a.d_in) * 2;
  g.xs[1] = static_cast<uint64_t>(a.d_in) * 2 * static_cast<uint64_t>(a.T);
  g.L = a.L;
  g.ld[0] = static_cast<uint64_t>(a.k);
  g.ld[1] = static_cast<uint64_t>(a.T);
  g.ld[2] = static_cast<uint64_t>(a.B);
  g.ls[0] = static_cast<uint64_t>(a.k) * 2;
  g.ls[1] = static_cast<uint64_t>(a.k) * 2 * static_cast<uint64_t>(a.T);
  g.d_in = a.d_in;
  g.k = a.k;
  g.rows = static_cast<int>(a.T);
  g.B = static_cast<int>(a.B);
  g.S = a.splits;
  g.Ts = a.split_rows;
  return g;
}

// The rank-k factor GEMM C^T = W_res Tb^T (d_out x B*k) from the K-major
// (B*k) x d_in operand Tb (with its low part Tlo when split_t), optionally
// also storing the low parts of C^T (Ctlo, hilo).
struct RFactorStage {
  const void* Tb;
  const void* Tlo;
  void* Ct;
  void* Ctlo;
  bool split_t, hilo;
  int smem_cap;
  unsigned long long* trace;
};

int launch_rfactor_stage(const RFactorStage& r, const Bf16Forward& a, const DeviceInfo& dev,
                         cudaStream_t s, bool pdl) {
  RFactorPolicy::Params p;
  const int Bk = static_cast<int>(a.B) * a.k;
  p.d_in = a.d_in;
  p.d_out = a.d_out;
  p.Bk = Bk;
  p.bn = std::min(256, (pick_bn(Bk) + 63) / 64 * 64);  // whole 64-column store boxes
  p.n_tiles_n = ceil_div(Bk, p.bn);
  uint64_t dw[2] = {static_cast<uint64_t>(a.d_in), static_cast<uint64_t>(a.d_out)};
  uint64_t sw[1] = {static_cast<uint64_t>(a.d_in) * 2};
  uint32_t bw[2] = {64, 128};
  if (!encode_tmap_bf16(&p.tmW, a.W_res, 2, dw, sw, bw, 128)) return -2;
  // Pairs halve each SM's share of T' per k-step; they need enough pair
  // tiles to keep the SMs busy and an even column tile.
  const bool rf_pairs = a.use_pairs && p.bn % 32 == 0 && p.bn >= 64 &&
                        ceil_div(a.d_out, 256) * p.n_tiles_n >= dev.sm_count / 4;
  uint64_t dt[2] = {static_cast<uint64_t>(a.d_in), static_cast<uint64_t>(Bk)};
  uint32_t bt[2] = {64, static_cast<uint32_t>(rf_pairs ? p.bn / 2 : p.bn)};
  if (!encode_tmap_bf16(&p.tmT, r.Tb, 2, dt, sw, bt, 128)) return -2;
  p.split_t = r.split_t ? 1 : 0;
  if (r.split_t) {
    if (!encode_tmap_bf16(&p.tmTlo, r.Tlo, 2, dt, sw, bt, 128)) return -2;
  } else {
    p.tmTlo = p.tmT;
  }
  const uint32_t parts = r.split_t ? 2u : 1u;  // B operands per stage
  uint64_t dc[2] = {static_cast<uint64_t>(Bk), static_cast<uint64_t>(a.d_out)};
  uint64_t sc[1] = {static_cast<uint64_t>(Bk) * 2};
  uint32_t bc[2] = {64, 128};
  if (!encode_tmap_bf16(&p.tmC, r.Ct, 2, dc, sc, bc, 128)) return -2;
  p.hilo = r.hilo ? 1 : 0;
  if (r.hilo) {
    if (!encode_tmap_bf16(&p.tmClo, r.Ctlo, 2, dc, sc, bc, 128)) return -2;
  } else {
    p.tmClo = p.tmC;
  }
  if (rf_pairs) {
    const int tiles = ceil_div(a.d_out, 256) * p.n_tiles_n;
    const uint32_t part_bytes = static_cast<uint32_t>(p.bn / 2) * 128u;
    const uint32_t smem =
        setup_common<RFactorPairPolicy>(p.c, tiles, 128 * 128, parts * part_bytes, p.bn, false,
                                        false, a.status, dev, r.smem_cap);
    if (!smem) return -3;
    p.c.b_parts = parts;
    p.c.b_part_desc = part_bytes >> 4;
    p.c.trigger_after_wait = 1;
    p.c.early = pdl ? 1 : 0;  // W_res before the wait
    p.c.idesc = idesc_bf16(256, p.bn, false, false);
    p.c.trace = r.trace;
    return launch_gemm_pair<RFactorPairPolicy>(p, smem, dev, s, pdl) ? -1 : 0;
  }
  const int tiles = ceil_div(a.d_out, 128) * p.n_tiles_n;
  const uint32_t part_bytes = static_cast<uint32_t>(p.bn) * 128u;
  const uint32_t smem =
      setup_common<RFactorPolicy>(p.c, tiles, 128 * 128, parts * part_bytes, p.bn, false, false,
                                  a.status, dev, r.smem_cap);
  if (!smem) return -3;
  p.c.b_parts = parts;
  p.c.b_part_desc = part_bytes >> 4;
  p.c.trigger_after_wait = 1;
  p.c.early = pdl ? 1 : 0;  // W_res before the wait
  p.c.trace = r.trace;
  return launch_gemm<RFactorPolicy>(p, smem, dev, s, pdl) ? -1 : 0;
}

// The static part of an output stage: Z (N x zcols) times U^T, dense (U is
// d_out x zcols) or block-diagonal (zb_w > 0: U holds zb_n blocks of zb_w
// rows x zb_k columns, K-major, and output block c takes Z's columns
// c*zb_k .. + zb_k: a Monarch factor).
struct OutStatic {
  const void* Z;
  int zcols;
  const void* U;
  int zb_w, zb_k, zb_n;
};

// The output stage Y = (static part) (+ bias) + sum_b mask_b(L) C_b with the
// correction's left factor L (N x k) and right factor C^T (d_out x B*k)
// (k = 0: the static part alone), with their low parts when hilo.
// early_static: the static operands are complete when this grid launches (it
// follows the correction chain, or a grid that does not trigger early), so
// they may be loaded before the dependency wait.
template <bool kExt, bool kBias>
int launch_out_as(OutParams& p, bool use_pairs, const Bf16Forward& a, const DeviceInfo& dev,
                  cudaStream_t s, bool pdl, bool early_static) {
  unsigned long long* tr = a.trace ? a.trace + 4 * kTraceCtas * kTraceSlots : nullptr;
  if (use_pairs) {
    using Pol = OutPairPolicyT<kExt, kBias>;
    const int tiles = ceil_div(p.N, 256) * p.n_tiles_n;
    const uint32_t smem = setup_common<Pol>(p.c, tiles, 128 * 128, (p.bn / 2) * 128, p.bn, false,
                                            false, a.status, dev);
    if (!smem) return -3;
    p.c.idesc = idesc_bf16(256, p.bn, false, false);
    p.c.trace = tr;
    p.c.early = pdl && early_static ? 1 : 0;
    return launch_gemm_pair<Pol>(p, smem, dev, s, pdl) ? -1 : 0;
  }
  using Pol = OutPolicyT<kExt, kBias>;
  const int tiles = ceil_div(p.N, 128) * p.n_tiles_n;
  const uint32_t smem =
      setup_common<Pol>(p.c, tiles, 128 * 128, p.bn * 128, p.bn, false, false, a.status, dev);
  if (!smem) return -3;
  p.c.trace = tr;
  p.c.early = pdl && early_static ? 1 : 0;
  return launch_gemm<Pol>(p, smem, dev, s, pdl) ? -1 : 0;
}

int launch_out_stage(const OutStatic& st, const void* L, const void* Llo, const void* Ct,
                     const void* Ctlo, bool hilo, int k, int d_out, void* Y, const void* bias,
                     const Bf16Forward& a, const DeviceInfo& dev, cudaStream_t s, bool pdl,
                     bool early_static = false) {
  const int64_t N = a.B * a.T;
  OutParams p;
  p.N = static_cast<int>(N);
  p.r = st.zcols;
  p.k = k;
  p.T = static_cast<int>(a.T);
  p.B = static_cast<int>(a.B);
  p.bn = d_out % 256 == 0 ? 256 : (d_out % 128 == 0 ? 128 : 64);
  if (d_out < p.bn) p.bn = 64;
  p.n_tiles_n = ceil_div(d_out, p.bn);
  p.zb_w = st.zb_w;
  p.zb_k = st.zb_k;
  p.zb_n = st.zb_n;
  p.nkz = st.zb_w > 0 ? ceil_div(st.zb_k, 64) : ceil_div(st.zcols, 64);
  p.nkl = k > 0 ? ceil_div(k, 64) : 0;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.d_out = d_out;

  uint64_t dz[2] = {static_cast<uint64_t>(st.zcols), static_cast<uint64_t>(N)};
  uint64_t sz[1] = {static_cast<uint64_t>(st.zcols) * 2};
  uint32_t bz[2] = {64, 128};
  if (!encode_tmap_bf16(&p.tmZ, st.Z, 2, dz, sz, bz, 128)) return -2;
  const bool use_pairs = a.use_pairs && p.bn >= 128;
  const uint32_t bbox = static_cast<uint32_t>(use_pairs ? p.bn / 2 : p.bn);
  if (st.zb_w > 0) {
    uint64_t du[3] = {static_cast<uint64_t>(st.zb_k), static_cast<uint64_t>(st.zb_w),
                      static_cast<uint64_t>(st.zb_n)};
    uint64_t su[2] = {static_cast<uint64_t>(st.zb_k) * 2,
                      static_cast<uint64_t>(st.zb_k) * 2 * static_cast<uint64_t>(st.zb_w)};
    uint32_t bu[3] = {64, bbox, 1};
    if (!encode_tmap_bf16(&p.tmU, st.U, 3, du, su, bu, 128)) return -2;
  } else {
    uint64_t du[2] = {static_cast<uint64_t>(st.zcols), static_cast<uint64_t>(d_out)};
    uint32_t bu[2] = {64, bbox};
    if (!encode_tmap_bf16(&p.tmU, st.U, 2, du, sz, bu, 128)) return -2;
  }
  p.narrow = k > 0 && k <= 32 ? 1 : 0;
  if (k > 0) {
    uint64_t dl[3] = {static_cast<uint64_t>(k), static_cast<uint64_t>(a.T),
                      static_cast<uint64_t>(a.B)};
    uint64_t sl[2] = {static_cast<uint64_t>(k) * 2,
                      static_cast<uint64_t>(k) * 2 * static_cast<uint64_t>(a.T)};
    const uint32_t kw = p.narrow ? 32u : 64u;  // box columns of the correction
    const int sw = p.narrow ? 64 : 128;
    uint32_t bl[3] = {kw, 128, 1};
    if (!encode_tmap_bf16(&p.tmL, L, 3, dl, sl, bl, sw)) return -2;
    const int64_t Bk = a.B * k;
    uint64_t dc[2] = {static_cast<uint64_t>(Bk), static_cast<uint64_t>(d_out)};
    uint64_t sc[1] = {static_cast<uint64_t>(Bk) * 2};
    uint32_t bc[2] = {kw, bbox};
    if (!encode_tmap_bf16(&p.tmC, Ct, 2, dc, sc, bc, sw)) return -2;
    if (hilo) {
      if (!encode_tmap_bf16(&p.tmLlo, Llo, 3, dl, sl, bl, sw)) return -2;
      if (!encode_tmap_bf16(&p.tmClo, Ctlo, 2, dc, sc, bc, sw)) return -2;
    } else {
      p.tmLlo = p.tmL;
      p.tmClo = p.tmC;
    }
  } else {
    p.tmL = p.tmZ;
    p.tmC = p.tmU;
    p.tmLlo = p.tmZ;
    p.tmClo = p.tmU;
  }
  p.hilo = k > 0 && hilo ? 1 : 0;
  uint64_t dy[2] = {static_cast<uint64_t>(d_out), static_cast<uint64_t>(N)};
  uint64_t sy[1] = {static_cast<uint64_t>(d_out) * 2};
  uint32_t by[2] = {64, 128};
  if (!encode_tmap_bf16(&p.tmY, Y, 2, dy, sy, by, 128)) return -2;
  // each layer takes the kernel compiled with only the options it uses
  const bool ext = p.hilo || p.zb_w > 0;
  if (p.bias != nullptr)
    return ext ? launch_out_as<true, true>(p, use_pairs, a, dev, s, pdl, early_static)
               : launch_out_as<false, true>(p, use_pairs, a, dev, s, pdl, early_static);
  return ext ? launch_out_as<true, false>(p, use_pairs, a, dev, s, pdl, early_static)
             : launch_out_as<false, false>(p, use_pairs, a, dev, s, pdl, early_static);
}

// P2_b = X_b (RW_b)^T over P2 (N x k), RW: (B*k) x d_in (XRwPolicy).
int launch_xrw_stage(const void* RW, void* P2, const Bf16Forward& a, const DeviceInfo& dev,
                     cudaStream_t s, bool pdl) {
  const int64_t N = a.B * a.T;
  XRwPolicy::Params p;
  p.N = static_cast<int>(N);
  p.d_in = a.d_in;
  p.k = a.k;
  p.kpad = ceil_div(a.k, 16) * 16;
  p.T = static_cast<int>(a.T);
  p.B = static_cast<int>(a.B);
  p.nkd = ceil_div(a.d_in, 64);
  p.P2 = static_cast<__nv_bfloat16*>(P2);
  uint64_t dx[3] = {static_cast<uint64_t>(a.d_in), static_cast<uint64_t>(a.T),
                    static_cast<uint64_t>(a.B)};
  uint64_t sx[2] = {static_cast<uint64_t>(a.d_in) * 2,
                    static_cast<uint64_t>(a.d_in) * 2 * static_cast<uint64_t>(a.T)};
  uint32_t bx[3] = {64, 128, 1};
  if (!encode_tmap_bf16(&p.tmX, a.X, 3, dx, sx, bx, 128)) return -2;
  uint64_t dr[2] = {static_cast<uint64_t>(a.d_in), static_cast<uint64_t>(a.B * a.k)};
  uint64_t sr[1] = {static_cast<uint64_t>(a.d_in) * 2};
  uint32_t br[2] = {64, static_cast<uint32_t>(p.kpad)};
  if (!encode_tmap_bf16(&p.tmRW, RW, 2, dr, sr, br, 128)) return -2;
  const int tiles = static_cast<int>(ceil_div(N, static_cast<int64_t>(128)));
  const uint32_t smem = setup_common<XRwPolicy>(p.c, tiles, 128 * 128,
                                                static_cast<uint32_t>(p.kpad) * 128, p.kpad,
                                                false, false, a.status, dev);
  if (!smem) return -3;
  return launch_gemm<XRwPolicy>(p, smem, dev, s, pdl) ? -1 : 0;
}

int launch_proj_stage(const Bf16Forward& a, int k_eff, const float* MD, int* counters,
                      const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  const int64_t N = a.B * a.T;
  const int rk = a.r + a.k;  // VPt rows always hold [V | P]
  ProjPolicy::Params p;
  const ProjShape ps =
      proj_shape(N, a.d_in, a.r, k_eff, a.use_pairs, dev.sm_count, a.proj_pair_min_tiles,
                 a.proj_bn);
  p.N = static_cast<int>(N);
  p.d_in = a.d_in;
  p.r = a.r;
  p.k = k_eff;
  p.tma_store = ps.tma_store;
  p.bn = ps.bn;
  p.n_tiles_n = ps.n_tiles_n;
  p.Z = static_cast<__nv_bfloat16*>(a.Z);
  p.L = static_cast<__nv_bfloat16*>(a.L);
  const bool records = p.k > 0 && MD && counters && factor_record_floats(p.k) > 0;
  p.cnt = records ? counters : nullptr;
  p.ncnt = static_cast<int>(a.B);
  p.ksplit = ps.ksplit;
  p.kper = ps.kper;
  uint64_t dx[2] = {static_cast<uint64_t>(a.d_in), static_cast<uint64_t>(N)};
  uint64_t sx[1] = {static_cast<uint64_t>(a.d_in) * 2};
  uint32_t bx[2] = {64, 128};
  if (!encode_tmap_bf16(&p.tmX, a.X, 2, dx, sx, bx, 128)) return -2;
  uint64_t dw[2] = {static_cast<uint64_t>(a.d_in), static_cast<uint64_t>(rk)};
  uint32_t bw[2] = {64, static_cast<uint32_t>(ps.pairs ? p.bn / 2 : p.bn)};
  if (!encode_tmap_bf16(&p.tmW, a.VPt, 2, dw, sx, bw, 128)) return -2;
  uint32_t bs[2] = {64, 128};
  if (a.r > 0) {
    uint64_t dz[2] = {static_cast<uint64_t>(a.r), static_cast<uint64_t>(N)};
    uint64_t sz[1] = {static_cast<uint64_t>(a.r) * 2};
    if (!encode_tmap_bf16(&p.tmZ, a.Z, 2, dz, sz, bs, 128)) return -2;
  }
  if (p.k > 0) {
    uint64_t dl[2] = {static_cast<uint64_t>(p.k), static_cast<uint64_t>(N)};
    uint64_t sl[1] = {static_cast<uint64_t>(p.k) * 2};
    if (!encode_tmap_bf16(&p.tmL, a.L, 2, dl, sl, bs, 128)) return -2;
  } else {
    p.tmL = p.tmZ;
  }
  if (a.r == 0) p.tmZ = p.tmL;  // no static columns (the projection of a Monarch plan)
  unsigned long long* tr = a.trace ? a.trace + 0 * kTraceCtas * kTraceSlots : nullptr;
  if (ps.pairs) {
    const uint32_t smem = setup_common<ProjPairPolicy>(p.c, ps.tiles, 128 * 128,
                                                       (p.bn / 2) * 128, p.bn, false, false,
                                                       a.status, dev);
    if (!smem) return -3;
    p.c.idesc = idesc_bf16(256, p.bn, false, false);
    p.c.trace = tr;
    p.c.early = pdl ? 1 : 0;  // [V | P]^T before the wait
    return launch_gemm_pair<ProjPairPolicy>(p, smem, dev, s, pdl) ? -1 : 0;
  }
  const uint32_t smem = setup_common<ProjPolicy>(p.c, ps.tiles * p.ksplit, 128 * 128,
                                                 p.bn * 128, p.bn, false, false, a.status, dev);
  if (!smem) return -3;
  // split-K keeps a 128 x bn fp32 partial in the operand stages
  if (p.ksplit > 1 && static_cast<size_t>(p.c.stages) * (p.c.a_stage_bytes + p.c.b_stage_bytes) <
                          static_cast<size_t>(128) * p.bn * 4)
    return -3;
  p.c.trace = tr;
  p.c.early = pdl ? 1 : 0;  // [V | P]^T before the wait
  return launch_gemm<ProjPolicy>(p, smem, dev, s, pdl, p.ksplit) ? -1 : 0;
}

// half_steps >= 3 alternating updates ([DyRA] Sec. 2.2, Eq. 4-5 with the
// ridge of footnote 2; Sec. 3.3 compares 1, 1.5 and 2 iterations), from
// Alg. 1's first left factor L = X P. Each right update is formed
// explicitly, R_b = (L_b^T L_b + lambda I)^-1 (L_b^T X_b) W_res^T: the Gram
// stage writes L_b^T X_b and L_b^T L_b in fp32, the solve applies the
// inverse from the left (T'_b, bf16) and the rank-k GEMM gives R^T = W_res
// T'^T. Each further left update is L_b = X_b (R_b W_res)^T (R_b R_b^T +
// lambda I)^-1: the Gram stage over (W_res, R_b^T), whose rows are the d_out
// output features, gives R_b W_res and R_b R_b^T, the X (R W_res)^T GEMM
// writes P2 over L, and the solve turns it into L in place. The output stage
// adds L_b R_b of the last pair; the correction weight alpha scales the last
// update. Stages follow one another in stream order.
int launch_bf16_als(const Bf16Forward& a, const DeviceInfo& dev, cudaStream_t s) {
  const bool pdl = false;
  const int k = a.k;
  auto mark = [&](int i) {
    if (a.stage_events) cudaEventRecord(a.stage_events[i], s);
  };
  mark(0);
  if (launch_proj_stage(a, k, nullptr, nullptr, dev, s, pdl)) return -1;
  mark(1);
  int splits2 = 1, rows2 = 64;
  gram_split(a.d_out, a.B, a.d_in, k, dev.sm_count, &splits2, &rows2);
  for (int h = 2; h <= a.half_steps; ++h) {
    const float w = h == a.half_steps ? a.alpha : 1.f;
    if (h % 2 == 0) {  // right update from the current L (over a.L)
      GramStage g = layer_gram(a);
      g.TGf = a.TG;
      if (launch_gram_stage(g, a.status, dev, s, pdl)) return -1;
      if (launch_solve<__nv_bfloat16>(a.TG, 1, a.B, k, a.d_in, a.lambda,
                                      static_cast<__nv_bfloat16*>(a.Tp), a.status, s, pdl,
                                      nullptr, w))
        return -1;
      RFactorStage r = {a.Tp, nullptr, a.Ct, nullptr, false, false, 0, nullptr};
      if (launch_rfactor_stage(r, a, dev, s, pdl)) return -1;
    } else {  // left update from the current R (R^T over a.Ct)
      GramStage g = {};
      g.X = a.W_res;
      g.xd[0] = static_cast<uint64_t>(a.d_in);
      g.xd[1] = static_cast<uint64_t>(a.d_out);
      g.xd[2] = 1;
      g.xs[0] = static_cast<uint64_t>(a.d_in) * 2;
      g.xs[1] = static_cast<uint64_t>(a.d_in) * 2 * static_cast<uint64_t>(a.d_out);
      g.x_inst_fixed = 1;
      g.L = a.Ct;  // R_b^T: element (j, b*k + i) of the d_out x B*k matrix
      g.ld[0] = static_cast<uint64_t>(k);
      g.ld[1] = static_cast<uint64_t>(a.d_out);
      g.ld[2] = static_cast<uint64_t>(a.B);
      g.ls[0] = static_cast<uint64_t>(a.B) * k * 2;
      g.ls[1] = static_cast<uint64_t>(k) * 2;
      g.d_in = a.d_in;
      g.k = k;
      g.rows = a.d_out;
      g.B = static_cast<int>(a.B);
      g.S = splits2;
      g.Ts = rows2;
      g.Tb = static_cast<__nv_bfloat16*>(a.Tp);  // R_b W_res
      g.G = a.TG;                                // R_b R_b^T
      if (launch_gram_stage(g, a.status, dev, s, pdl)) return -1;
      if (launch_xrw_stage(a.Tp, a.L, a, dev, s, pdl)) return -1;
      if (launch_ltilde(a.TG, a.L, nullptr, nullptr, nullptr, 0, a.B, a.T, k, a.lambda, w,
                        a.status, s, pdl, /*defer_wait=*/false, nullptr))
        return -1;
    }
  }
  mark(2);
  mark(3);
  mark(4);
  const OutStatic st = {a.Z, a.r, a.U, 0, 0, 0};
  if (launch_out_stage(st, a.L, nullptr, a.Ct, nullptr, false, k, a.d_out, a.Y, a.bias, a, dev, s,
                       pdl))
    return -1;
  mark(5);
  return 0;
}

}  // namespace

namespace {

void mark_stage(const Bf16Forward& a, int i, cudaStream_t s) {
  if (a.stage_events) cudaEventRecord(a.stage_events[i], s);
}

// The correction of the one-step layer after the projection: the Gram stage,
// the rank-k factor GEMM Q = T W_res^T and, beside it, the solve L~ = L G^-1
// over L (programmatic dependent launches throughout).
int launch_correction(const Bf16Forward& a, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  GramStage g = layer_gram(a);
  g.Tb = static_cast<__nv_bfloat16*>(a.Tp);
  g.Tlo = a.split_t ? static_cast<__nv_bfloat16*>(a.Tplo) : nullptr;
  g.G = a.TG;
  g.trace = a.trace ? a.trace + 1 * kTraceCtas * kTraceSlots : nullptr;
  g.wait_ns = a.gram_wait_ns;
  if (launch_gram_stage(g, a.status, dev, s, pdl)) return -1;
  mark_stage(a, 2, s);
  // Q = T W_res^T needs the Gram stage's T only. The solve is launched
  // after it and runs beside it: this grid lets the solve start once its
  // own wait for the Gram stage is over, and its shared memory leaves room
  // on every SM for one solve block.
  RFactorStage r;
  r.Tb = a.Tp;
  r.Tlo = a.Tplo;
  r.Ct = a.Ct;
  r.Ctlo = a.Ctlo;
  r.split_t = a.split_t;
  r.hilo = a.hilo;
  r.smem_cap =
      dev.smem_per_sm > 0 && a.k <= 64
          ? dev.smem_per_sm - 2 * dev.smem_reserved - static_cast<int>(ltilde_smem_bytes(a.k))
          : 0;
  r.trace = a.trace ? a.trace + 3 * kTraceCtas * kTraceSlots : nullptr;
  if (launch_rfactor_stage(r, a, dev, s, pdl)) return -1;
  mark_stage(a, 3, s);
  // ------------------------------------------------------------- solve
  // L~ = L G^-1 over L, beside the GEMM for Q: it reads what the Gram
  // stage wrote and waits for the GEMM only before its blocks exit, so that
  // the output stage can rely on both. Every block factors its G_b while
  // that fits the SMs; beyond, the instance's first block factors it for
  // the others.
  const bool records = a.MD && a.counters && factor_record_floats(a.k) > 0;
  int mode = a.factor_mode;
  if (mode < 0)
    mode = a.B * ceil_div(a.T, static_cast<int64_t>(ltilde_rows_per_block(a.k))) > dev.sm_count
               ? 1
               : 0;
  if (!records) mode = 0;
  if (a.solver == 1) {
    // Newton-Schulz: one kernel inverts every G_b + lambda I and publishes
    // the records (it starts once the GEMM for Q is complete); every solve
    // block then reads its instance's record
    if (!records) return -1;
    if (launch_ns_inverse(a.TG, a.B, a.k, a.lambda, a.ns_iters, a.MD, a.counters, a.status, s))
      return -1;
    mode = 2;
  }
  return launch_ltilde(a.TG, a.L, a.hilo ? a.Llo : nullptr, a.MD, a.counters, mode, a.B, a.T,
                       a.k, a.lambda, a.alpha, a.status, s, pdl, /*defer_wait=*/true,
                       a.trace ? a.trace + 2 * kTraceCtas * kTraceSlots : nullptr)
             ? -1
             : 0;
}

// Monarch static part ([DyRA] App. B, square or rectangular blocks) under
// the same correction. The static product is two block-diagonal GEMMs on
// the output stage's kernel, each behind a shuffle of its input's columns
// (b1 b2 = d_in, b1' b2' = d_out, b2 b1' intermediate columns):
//   Xs[row][j2 b1 + m1]  = X[row][m1 b2 + j2]                      (shuffle)
//   M[row][j2 b1' + j1]  = sum_m1 Xs[row][j2 b1 + m1] L_j2[m1][j1]  (b2 blocks)
//   Ms[row][j1 b2 + j2]  = M[row][j2 b1' + j1]                      (shuffle)
//   Y[row][j1 b2' + i2]  = sum_j2 Ms[row][j1 b2 + j2] R_j1[j2][i2]  (b1' blocks)
//                          + bias + the correction's L~ Q segments
// The first three run in stream order; the correction chain follows with
// programmatic dependent launches, and the last GEMM takes its segments.
int launch_bf16_monarch(const Bf16Forward& a, const DeviceInfo& dev, cudaStream_t s) {
  const int64_t N = a.B * a.T;
  const int k = a.weight_only ? 0 : a.k;
  const int nmid = a.mb2 * a.mb1o;
  mark_stage(a, 0, s);
  if (launch_grid_transpose(a.X, a.Xs, N, a.mb1, a.mb2, dev.sm_count, s)) return -1;
  const OutStatic st1 = {a.Xs, a.d_in, a.Lt, a.mb1o, a.mb1, a.mb2};
  if (launch_out_stage(st1, nullptr, nullptr, nullptr, nullptr, false, 0, nmid, a.Ms, nullptr, a,
                       dev, s, false))
    return -1;
  if (launch_grid_transpose(a.Ms, a.Xs, N, a.mb2, a.mb1o, dev.sm_count, s)) return -1;
  mark_stage(a, 1, s);
  if (k > 0) {
    if (launch_proj_stage(a, k, a.MD, a.counters, dev, s, true)) return -1;
    if (launch_correction(a, dev, s, true)) return -1;
  } else {
    mark_stage(a, 2, s);
    mark_stage(a, 3, s);
  }
  mark_stage(a, 4, s);
  const OutStatic st2 = {a.Xs, nmid, a.Rt, a.mb2o, a.mb2, a.mb1o};
  if (launch_out_stage(st2, a.L, nullptr, a.Ct, nullptr, false, k, a.d_out, a.Y, a.bias, a, dev,
                       s, true, /*early_static=*/true))
    return -1;
  mark_stage(a, 5, s);
  return 0;
}

}  // namespace

int launch_bf16_forward(const Bf16Forward& a, const DeviceInfo& dev, cudaStream_t s) {
  const int64_t N = a.B * a.T;
  if (N == 0) return 0;
  if (a.Lt != nullptr) return launch_bf16_monarch(a, dev, s);
  const int k = a.weight_only ? 0 : a.k;
  if (k > 0 && a.half_steps > 2) return launch_bf16_als(a, dev, s);
  const bool pdl = true;
  mark_stage(a, 0, s);
  if (launch_proj_stage(a, k, a.MD, a.counters, dev, s, pdl)) return -1;
  mark_stage(a, 1, s);
  if (k > 0) {
    if (launch_correction(a, dev, s, pdl)) return -1;
  } else {
    mark_stage(a, 2, s);
    mark_stage(a, 3, s);
  }
  mark_stage(a, 4, s);
  const OutStatic st = {a.Z, a.r, a.U, 0, 0, 0};
  if (launch_out_stage(st, a.L, a.Llo, a.Ct, a.Ctlo, a.hilo, k, a.d_out, a.Y, a.bias, a, dev, s,
                       pdl, /*early_static=*/k > 0))
    return -1;
  mark_stage(a, 5, s);
  return 0;
}

}  // namespace dyra
