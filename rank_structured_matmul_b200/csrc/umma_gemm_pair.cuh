// umma_gemm_pair.cuh - the persistent GEMM skeleton on CTA pairs
// (tcgen05 .cta_group::2): a cluster of two CTAs computes a 256 x N tile
// with one MMA stream. Each CTA loads its 128 rows of A and N/2 rows of B, so
// per SM the operand traffic of a 128 x N output is a third lower than with
// one CTA per tile (A 128 x K plus B N/2 x K instead of B N x K).
//
// Roles as in umma_gemm.cuh (warp 0 producer, warp 1 MMA, warps 2..5
// epilogue), with these differences:
//  - both CTAs' copies complete on the leader's (even CTA's) full barrier;
//    only the leader arms it with the pair's byte count;
//  - only the leader's warp 1 issues MMAs; completions are committed to the
//    matching barrier of both CTAs (slot free, accumulator ready);
//  - both CTAs' epilogue warps (8) arrive on the leader's accumulator-free
//    barrier;
//  - TMEM is allocated and freed pairwise; the cluster synchronises after
//    set-up and before teardown.
// Waits are bounded as in the single-CTA skeleton.
//
// A pair policy supplies the single-CTA policy interface with `rank` added
// to load() (which CTA of the pair loads) and EpiCtx::rank set for the
// epilogue.
#pragma once

#include "umma_gemm.cuh"

namespace dyra {

template <class Pol>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    __maxnreg__(MaxRegs<Pol>::value)
    umma_gemm_pair_kernel(const __grid_constant__ typename Pol::Params p) {
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
  auto full_bar = [&](int s) { return sBar + 8u * s; };
  auto empty_bar = [&](int s) { return sBar + 8u * (kMaxStages + s); };
  auto tfull_bar = [&](int i) { return sBar + 8u * (2 * kMaxStages + i); };
  auto tempty_bar = [&](int i) { return sBar + 8u * (2 * kMaxStages + 2 + i); };
  const uint32_t fin_bar = sBar + 8u * (2 * kMaxStages + 4);
  uint32_t* tmem_slot =
      reinterpret_cast<uint32_t*>(smem + (sBar - sbase) + 8 * (2 * kMaxStages + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
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
      mbar_init(tempty_bar(i), 8);  // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(fin_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) Pol::prefetch(p);
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), c.tmem_cols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tr && threadIdx.x == 0) tr[kTrSetup] = globaltimer_ns();

  // Every CTA of this grid is resident (grid <= SMs), so the next kernel in
  // the stream may be launched now: its CTAs take SMs as ours leave and wait
  // in pdl_wait() for our results. This hides launch and set-up latency.
  // early: as in the single-CTA skeleton (the producer waits after its first
  // copies, the epilogue before its first output, the MMA warp never)
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
          if (pair < c.num_tiles) {
            Pol::decode(p, pair, t0);
            pre = min(S, Pol::kiters(p, t0));
          }
          for (int it = 0; it < pre; ++it) {  // fresh slots: nothing to wait for
            if (leader)
              mbar_arrive_expect_tx(full_bar(it), 2u * stage_tx<Pol>(p, t0, it));
            Pol::load_early(p, t0, it, sA + it * c.a_stage_bytes, sB + it * c.b_stage_bytes,
                            full_bar(it), rank);
          }
          pdl_wait();
          if (c.trigger_after_wait) pdl_launch_dependents();
          for (int it = 0; it < pre; ++it) {
            Pol::load_late(p, t0, it, sA + it * c.a_stage_bytes, sB + it * c.b_stage_bytes,
                           full_bar(it), rank);
            issued |= 1u << it;
            last_phase[it] = 0;
          }
          stage = pre % S;
          phase = pre == S ? 1u : 0u;
        }
      }
      for (int tile = pair; ok && tile < c.num_tiles; tile += npairs) {
        typename Pol::Tile t;
        Pol::decode(p, tile, t);
        const int nk = Pol::kiters(p, t);
        for (int it = tile == pair ? pre : 0; it < nk; ++it) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, w)) {
            ok = false;
            break;
          }
          if (leader)
            mbar_arrive_expect_tx(full_bar(stage), 2u * stage_tx<Pol>(p, t, it));
          Pol::load(p, t, it, sA + stage * c.a_stage_bytes, sB + stage * c.b_stage_bytes,
                    full_bar(stage), rank);
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
    if (leader && elect_one_sync()) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      const uint32_t idesc = c.idesc;
      const uint64_t da = Pol::adesc(p, sA, 1) - Pol::adesc(p, sA, 0);
      const uint64_t db = Pol::bdesc(p, sB, 1) - Pol::bdesc(p, sB, 0);
      uint32_t a = sA, b = sB;  // this stage's operands
      for (int tile = pair; tile < c.num_tiles; tile += npairs, ++local) {
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
          issue_stage<true>(d, a0, da, b0, db, idesc, ks, it == 0);
          if constexpr (HasBParts<Pol>::value)
            for (uint32_t part = 1; part < c.b_parts; ++part)
              issue_stage<true>(d, a0, da, b0 + part * c.b_part_desc, db, idesc, ks, false);
          mma_commit_pair(empty_bar(stage));
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
        mma_commit_pair(tfull_bar(acc));
        if (tr) {
          tr[kTrLastCommit] = globaltimer_ns();
          if (local < kTrProducerDone - kTrTileMma) tr[kTrTileMma + local] = globaltimer_ns();
        }
      }
      mma_commit_pair(fin_bar);
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
    e.rank = static_cast<int>(rank);
    e.tr = tr;
    int local = 0;
    for (int tile = pair; tile < c.num_tiles; tile += npairs, ++local) {
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
      if (lane == 0) mbar_arrive_leader(tempty_bar(acc));
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
  if (c.defer_wait) pdl_wait();
  block_sync_all();
  // Every copy issued has landed before either CTA leaves. The leader's full
  // barriers also count the other CTA's copies, and its MMA thread waited for
  // each of them in a normal run, so only a leader that gave up early drains
  // here, before the cluster barrier that holds the other CTA.
  if (leader && warp == 0 && issued && *abort_flag) {
    const unsigned long long deadline = globaltimer_ns() + kWaitLimitNs;
    for (int s = 0; s < S; ++s)
      if (issued & (1u << s)) (void)mbar_wait_until(full_bar(s), last_phase[s], deadline);
  }
  cluster_sync_all();  // the leader's MMAs into both TMEMs are complete
  if (tr && threadIdx.x == 0) tr[kTrExit] = globaltimer_ns();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, c.tmem_cols);
  }
}

}  // namespace dyra
