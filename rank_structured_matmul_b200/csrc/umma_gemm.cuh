// umma_gemm.cuh - persistent, warp-specialised tcgen05 GEMM skeleton.
//
// One CTA per SM (grid = min(tiles, SMs)), 192 threads:
//   warp 0      TMA producer: fills a ring of `stages` shared-memory slots
//   warp 1      MMA issuer: one elected thread issues tcgen05.mma (M = 128)
//               into one of two TMEM accumulators, and owns the TMEM allocation
//   warps 2..5  epilogue: tcgen05.ld the finished accumulator (warp w reads
//               TMEM lanes 32*(w%4) .. +31, i.e. those rows of the tile) and
//               hand the values to the policy's epilogue
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1. Every barrier wait is bounded (sm100::mbar_wait); on a timeout the CTA
// raises its status word, drains the copies and MMAs it issued, frees TMEM and
// returns.
//
// A policy `Pol` supplies:
//   struct Params { GemmCommon c; ... };
//   struct Tile { ... };
//   static void decode(const Params&, int tile, Tile&);
//   static int  kiters(const Params&, const Tile&);
//   static void load(const Params&, const Tile&, int it, uint32_t sa, uint32_t sb, uint32_t bar);
//   static int  ksteps(const Params&, const Tile&, int it);        // K16 MMAs in slot
//   static uint64_t adesc(const Params&, uint32_t sa, int ks);
//   static uint64_t bdesc(const Params&, uint32_t sb, int ks);
//   static void epilogue(const Params&, const Tile&, uint32_t tacc, EpiCtx&);
//   static void epilogue_drain(const Params&, EpiCtx&);
//   static void prefetch(const Params&);
//   static constexpr uint32_t kEpiSmemBytes;
#pragma once

#include <type_traits>

#include "internal.h"
#include "sm100.cuh"

namespace dyra {

constexpr int kGemmThreads = 192;
constexpr int kMaxStages = 8;

// Optional timeline: when GemmCommon::trace is set, each CTA writes
// %globaltimer (ns) into trace[blockIdx.x * kTraceSlots + slot]
// (kTraceSlots is defined in internal.h).
enum TraceSlot {
  kTrEntry = 0,        // kernel entry
  kTrSetup = 1,        // barriers initialised, TMEM allocated
  kTrDepsReady = 2,    // the previous grid's results are visible
  kTrFirstIssue = 3,   // producer issued its first copy
  kTrLastIssue = 4,    // producer issued its last copy
  kTrFirstData = 5,    // MMA thread saw its first full slot
  kTrLastCommit = 6,   // MMA thread committed its last tile
  kTrEpiFirst = 7,     // epilogue saw its first finished accumulator
  kTrExit = 8,         // all roles done, before TMEM is freed
  kTrTileDone = 9,     // + i: epilogue finished its i-th tile (i < 27)
  kTrTileMma = 36,     // + i: MMA thread committed its i-th tile (i < 20)
  kTrProducerDone = 56,  // producer's copies all landed
  kTrMmaDone = 57,       // MMA thread's last MMA complete
  kTrEpiDone = 58,       // epilogue warps done (before the closing barrier)
  kTrSplitWritten = 60,  // split-K: partial tile written and fenced
  kTrSplitArrived = 61,  // split-K: every split of the tile has arrived
  kTrSplitReduced = 62   // split-K: this split's slice is reduced and stored
};

struct GemmCommon {
  int num_tiles;
  int stages;
  uint32_t a_stage_bytes;
  uint32_t b_stage_bytes;
  uint32_t acc_cols;   // TMEM columns of one accumulator (>= MMA N)
  uint32_t tmem_cols;  // allocated columns: power of two >= 2 * acc_cols, >= 32
  uint32_t idesc;      // instruction descriptor (M = 128, N, majors)
  int* status;         // device status word
  unsigned long long* trace;  // optional timeline, nullptr when off
  // 1: the operands do not depend on the grid launched just before this one
  // (they depend on an earlier grid, complete once the previous grid's blocks
  // have started); this grid then waits for the previous one only before it
  // exits, so that the next grid can still rely on both.
  int defer_wait;
  // 1: the next grid may start only once this grid's own dependency wait is
  // over (that grid then relies on what the grid before this one wrote).
  int trigger_after_wait;
  // B operands per stage (1, or 2 when a second operand, e.g. the low part of
  // a split bf16 value, accumulates into the same tile with the same A), and
  // the smem descriptor step from one part to the next
  uint32_t b_parts;
  uint64_t b_part_desc;
  // limit of one pipeline wait in ns (sm100::kWaitLimitNs; a diagnostic may
  // shorten it to make a wait run out). Drains keep kWaitLimitNs.
  unsigned long long wait_ns;
  // 1: the producer issues the operands of the first tile's first stages that
  // do not depend on earlier grids (Pol::load_early) before the dependency
  // wait, and the rest (Pol::load_late) after it; only the producer and the
  // epilogue wait. Policies opt in with kEarly.
  int early;
};

// Issues one stage's ks MMAs (K = 16 each) back to back. The tensor pipe idles
// whenever an MMA is issued late, even by a few dozen cycles of address
// arithmetic (a runtime k-step loop measured 168 cycles per M=256, N=256 MMA
// instead of 128), so the descriptors advance by a fixed step (their address
// field is linear in the k-step) and the usual counts are unrolled.
template <bool PAIR>
__device__ __forceinline__ void issue_stage(uint32_t d, uint64_t a0, uint64_t da, uint64_t b0,
                                            uint64_t db, uint32_t idesc, int ks, bool first) {
  auto mma = [&](uint64_t ad, uint64_t bd, uint32_t accum) {
    if constexpr (PAIR)
      sm100::mma_bf16_pair(d, ad, bd, idesc, accum);
    else
      sm100::mma_bf16(d, ad, bd, idesc, accum);
  };
  const uint32_t acc0 = first ? 0u : 1u;
  if (ks == 4) {
    mma(a0, b0, acc0);
    mma(a0 + da, b0 + db, 1u);
    mma(a0 + 2 * da, b0 + 2 * db, 1u);
    mma(a0 + 3 * da, b0 + 3 * db, 1u);
  } else if (ks == 2) {
    mma(a0, b0, acc0);
    mma(a0 + da, b0 + db, 1u);
  } else {
    for (int k = 0; k < ks; ++k) mma(a0 + k * da, b0 + k * db, k == 0 ? acc0 : 1u);
  }
}

struct EpiCtx {
  int row;            // tile row owned by this thread, 0..127
  int lane;           // lane in warp
  int quad;           // TMEM lane quadrant of this warp
  int tid;            // 0..127 among the epilogue threads
  uint8_t* smem;      // policy scratch (kEpiSmemBytes), 1024-byte aligned
  uint32_t smem_u32;  // same, as a shared-window address
  uint32_t counter;   // running counter the policy may use (e.g. store buffers)
  int rank;           // CTA of the pair (0 for single-CTA kernels)
  unsigned long long* tr;  // this CTA's timeline row, or nullptr
  uint8_t* stage;          // the operand stages (free once the CTA's last MMA is complete)
  uint32_t stage_u32;
  uint32_t stage_bytes;
};

__host__ __device__ inline uint32_t gemm_smem_bytes(int stages, uint32_t a_bytes,
                                                    uint32_t b_bytes, uint32_t epi_bytes) {
  // 1024 alignment slack + stages + epilogue scratch + barriers/slots
  return 1024u + static_cast<uint32_t>(stages) * (a_bytes + b_bytes) + epi_bytes + 256u;
}

// Register cap of a policy's kernel: Pol::kMaxRegs if it declares one (a
// GEMM that must share its SMs with another kernel's blocks), else the
// hardware limit.
template <class Pol, class = void>
struct MaxRegs {
  static constexpr int value = 255;
};
template <class Pol>
struct MaxRegs<Pol, std::void_t<decltype(Pol::kMaxRegs)>> {
  static constexpr int value = Pol::kMaxRegs;
};

// Whether a policy can split its first stages' copies around the dependency
// wait (Pol::kEarly, with load_early / load_late).
template <class Pol, class = void>
struct HasEarly {
  static constexpr bool value = false;
};
template <class Pol>
struct HasEarly<Pol, std::void_t<decltype(Pol::kEarly)>> {
  static constexpr bool value = Pol::kEarly;
};

// Whether a policy may run with more than one B operand per stage
// (Pol::kBParts; GemmCommon::b_parts is 1 for the others).
template <class Pol, class = void>
struct HasBParts {
  static constexpr bool value = false;
};
template <class Pol>
struct HasBParts<Pol, std::void_t<decltype(Pol::kBParts)>> {
  static constexpr bool value = Pol::kBParts;
};

// Stages of different layouts (Pol::kStageLayouts): the policy gives each
// stage's byte count and its first shared memory descriptors; otherwise every
// stage holds a_stage_bytes + b_stage_bytes in the policy's one layout.
template <class Pol, class = void>
struct HasStageLayouts {
  static constexpr bool value = false;
};
template <class Pol>
struct HasStageLayouts<Pol, std::void_t<decltype(Pol::kStageLayouts)>> {
  static constexpr bool value = Pol::kStageLayouts;
};
template <class Pol>
__device__ __forceinline__ uint32_t stage_tx(const typename Pol::Params& p,
                                             const typename Pol::Tile& t, int it) {
  if constexpr (HasStageLayouts<Pol>::value)
    return Pol::stage_tx(p, t, it);
  else
    return p.c.a_stage_bytes + p.c.b_stage_bytes;
}
template <class Pol>
__device__ __forceinline__ uint64_t stage_adesc(const typename Pol::Params& p,
                                                const typename Pol::Tile& t, int it, uint32_t a) {
  if constexpr (HasStageLayouts<Pol>::value)
    return Pol::stage_adesc(p, t, it, a);
  else
    return Pol::adesc(p, a, 0);
}
template <class Pol>
__device__ __forceinline__ uint64_t stage_bdesc(const typename Pol::Params& p,
                                                const typename Pol::Tile& t, int it, uint32_t b) {
  if constexpr (HasStageLayouts<Pol>::value)
    return Pol::stage_bdesc(p, t, it, b);
  else
    return Pol::bdesc(p, b, 0);
}

template <class Pol>
__global__ void __launch_bounds__(kGemmThreads, 1) __maxnreg__(MaxRegs<Pol>::value)
    umma_gemm_kernel(const __grid_constant__ typename Pol::Params p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const GemmCommon& c = p.c;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const int S = c.stages;
  const uint32_t sA = sbase;
  const uint32_t sB = sA + static_cast<uint32_t>(S) * c.a_stage_bytes;
  const uint32_t sEpi = sB + static_cast<uint32_t>(S) * c.b_stage_bytes;
  const uint32_t sBar = sEpi + Pol::kEpiSmemBytes;
  // barriers: full[S], empty[S], tfull[2], tempty[2], fin
  auto full_bar = [&](int s) { return sBar + 8u * s; };
  auto empty_bar = [&](int s) { return sBar + 8u * (kMaxStages + s); };
  auto tfull_bar = [&](int i) { return sBar + 8u * (2 * kMaxStages + i); };
  auto tempty_bar = [&](int i) { return sBar + 8u * (2 * kMaxStages + 2 + i); };
  const uint32_t fin_bar = sBar + 8u * (2 * kMaxStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (sBar - sbase) + 8 * (2 * kMaxStages + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  unsigned long long* const tr =
      c.trace && blockIdx.x < kTraceCtas ? c.trace + blockIdx.x * kTraceSlots : nullptr;
  if (tr && threadIdx.x == 0) tr[kTrEntry] = globaltimer_ns();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 4);
    }
    mbar_init(fin_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) Pol::prefetch(p);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), c.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tr && threadIdx.x == 0) tr[kTrSetup] = globaltimer_ns();
  // Inputs written by the previous kernel in the stream are visible from here.
  // Every CTA of this grid is resident (grid <= SMs), so the next kernel in
  // the stream may be launched now: its CTAs take SMs as ours leave and wait
  // in pdl_wait() for our results. This hides launch and set-up latency.
  // early: the producer waits after its first copies, the epilogue before
  // its first output, and the MMA warp (shared memory and TMEM only) never.
  const bool early = HasEarly<Pol>::value && c.early && !c.defer_wait;
  if (!c.trigger_after_wait) pdl_launch_dependents();
  if (!c.defer_wait && !early) pdl_wait();
  if (c.trigger_after_wait && !early) pdl_launch_dependents();
  if (tr && threadIdx.x == 0) tr[kTrDepsReady] = globaltimer_ns();

  WaitCtx w{abort_flag, c.status, c.wait_ns};
  // producer state kept for the drain after the closing barrier
  uint32_t last_phase[kMaxStages];
  uint32_t issued = 0;

  if (warp == 0) {
    if (elect_one_sync()) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int pre = 0;  // stages of the first tile issued around the dependency wait
      if constexpr (HasEarly<Pol>::value) {
        if (early) {
          typename Pol::Tile t0;
          if (blockIdx.x < c.num_tiles) {
            Pol::decode(p, blockIdx.x, t0);
            pre = min(S, Pol::kiters(p, t0));
          }
          for (int it = 0; it < pre; ++it) {  // fresh slots: nothing to wait for
            mbar_arrive_expect_tx(full_bar(it), stage_tx<Pol>(p, t0, it));
            Pol::load_early(p, t0, it, sA + it * c.a_stage_bytes, sB + it * c.b_stage_bytes,
                            full_bar(it));
          }
          pdl_wait();
          if (c.trigger_after_wait) pdl_launch_dependents();
          for (int it = 0; it < pre; ++it) {
            Pol::load_late(p, t0, it, sA + it * c.a_stage_bytes, sB + it * c.b_stage_bytes,
                           full_bar(it));
            issued |= 1u << it;
            last_phase[it] = 0;
          }
          stage = pre % S;
          phase = pre == S ? 1u : 0u;
        }
      }
      for (int tile = blockIdx.x; ok && tile < c.num_tiles; tile += gridDim.x) {
        typename Pol::Tile t;
        Pol::decode(p, tile, t);
        const int nk = Pol::kiters(p, t);
        for (int it = tile == static_cast<int>(blockIdx.x) ? pre : 0; it < nk; ++it) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, w)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), stage_tx<Pol>(p, t, it));
          Pol::load(p, t, it, sA + stage * c.a_stage_bytes, sB + stage * c.b_stage_bytes,
                    full_bar(stage));
          if (tr) {
            if (!issued) tr[kTrFirstIssue] = globaltimer_ns();
            tr[kTrLastIssue] = globaltimer_ns();
          }
          issued |= 1u << stage;
          last_phase[stage] = phase;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (tr) tr[kTrProducerDone] = globaltimer_ns();
    }
  } else if (warp == 1) {
    if (elect_one_sync()) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      const uint32_t idesc = c.idesc;
      const uint64_t da = Pol::adesc(p, sA, 1) - Pol::adesc(p, sA, 0);
      const uint64_t db = Pol::bdesc(p, sB, 1) - Pol::bdesc(p, sB, 0);
      uint32_t a = sA, b = sB;  // this stage's operands
      for (int tile = blockIdx.x; tile < c.num_tiles; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, w)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc) * c.acc_cols;
        typename Pol::Tile t;
        Pol::decode(p, tile, t);
        const int nk = Pol::kiters(p, t);
        bool ok = true;
        for (int it = 0; it < nk; ++it) {
          // what the stage's MMAs need besides its data, before the wait
          const int ks = Pol::ksteps(p, t, it);
          const uint64_t a0 = stage_adesc<Pol>(p, t, it, a), b0 = stage_bdesc<Pol>(p, t, it, b);
          if (!mbar_wait(full_bar(stage), phase, w)) {
            ok = false;
            break;
          }
          if (tr && local == 0 && it == 0) tr[kTrFirstData] = globaltimer_ns();
          tc_fence_after();
          issue_stage<false>(d, a0, da, b0, db, idesc, ks, it == 0);
          if constexpr (HasBParts<Pol>::value)
            for (uint32_t part = 1; part < c.b_parts; ++part)
              issue_stage<false>(d, a0, da, b0 + part * c.b_part_desc, db, idesc, ks, false);
          mma_commit(empty_bar(stage));
          a += c.a_stage_bytes;
          b += c.b_stage_bytes;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
            a = sA;
            b = sB;
          }
        }
        if (!ok) break;
        mma_commit(tfull_bar(acc));
        if (tr) {
          tr[kTrLastCommit] = globaltimer_ns();
          if (local < kTrProducerDone - kTrTileMma) tr[kTrTileMma + local] = globaltimer_ns();
        }
      }
      // All MMAs issued by this thread are complete before TMEM is freed.
      mma_commit(fin_bar);
      (void)mbar_wait_until(fin_bar, 0, globaltimer_ns() + kWaitLimitNs);
      if (tr) tr[kTrMmaDone] = globaltimer_ns();
    }
  } else {
    if (early) pdl_wait();
    EpiCtx e;
    e.quad = warp & 3;
    e.lane = lane;
    e.row = e.quad * 32 + lane;
    e.tid = threadIdx.x - 64;
    e.smem = smem + (sEpi - sbase);
    e.smem_u32 = sEpi;
    e.counter = 0;
    e.rank = 0;
    e.tr = tr;
    e.stage = smem;
    e.stage_u32 = sA;
    e.stage_bytes = static_cast<uint32_t>(S) * (c.a_stage_bytes + c.b_stage_bytes);
    int local = 0;
    for (int tile = blockIdx.x; tile < c.num_tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(tfull_bar(acc), acc_phase, w)) break;
      tc_fence_after();
      if (tr && e.tid == 0 && local == 0) tr[kTrEpiFirst] = globaltimer_ns();
      typename Pol::Tile t;
      Pol::decode(p, tile, t);
      const uint32_t tacc = tmem + static_cast<uint32_t>(acc) * c.acc_cols +
                            (static_cast<uint32_t>(e.quad * 32) << 16);
      Pol::epilogue(p, t, tacc, e);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (tr && e.tid == 0 && local < kTrTileMma - kTrTileDone)
        tr[kTrTileDone + local] = globaltimer_ns();
    }
    Pol::epilogue_drain(p, e);
    if (tr && e.tid == 0) tr[kTrEpiDone] = globaltimer_ns();
  }
  // Warps 0 and 1 ran their roles on one elected lane: reconverge them
  // before the closing barrier (which counts threads, so it holds the block
  // until the epilogue warps are done with TMEM either way).
  __syncwarp();
  // A policy whose tiles end in a cluster-wide step (split-K partials summed
  // over distributed shared memory) runs it here: every CTA of the cluster has
  // finished its tile when the first barrier opens, and none leaves before
  // the others have read its shared memory.
  if (Pol::cluster_finish(p)) {
    cluster_sync_all();
    if (warp >= 2) Pol::finish(p, threadIdx.x - 64, sA, tr);
    cluster_sync_all();
  }
  if (c.defer_wait) pdl_wait();
  block_sync_all();
  // Every copy the producer issued has landed before the CTA leaves: in a
  // normal run the MMA thread waited for each of them, so only a run that
  // gave up early drains here (one shared deadline for all slots).
  if (warp == 0 && issued && *abort_flag) {
    const unsigned long long deadline = globaltimer_ns() + kWaitLimitNs;
    for (int s = 0; s < S; ++s)
      if (issued & (1u << s)) (void)mbar_wait_until(full_bar(s), last_phase[s], deadline);
  }
  if (tr && threadIdx.x == 0) tr[kTrExit] = globaltimer_ns();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, c.tmem_cols);
  }
}

}  // namespace dyra
