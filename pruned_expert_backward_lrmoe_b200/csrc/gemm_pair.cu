// a4 for bf16 storage on pairs of SMs: the variable-size grouped GEMMs with one
// tcgen05 MMA shared by the two CTAs of a cluster.
//
// "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE", bullet 5
// (German page, paragraph 4: "gruppierte GEMMs variabler Größe"): the expert
// gradients are grouped GEMMs over the compacted per-expert blocks, with no
// zero padding.
//
// Same tiles and epilogues as grouped_gemm_tc in gemm_tc.cu, but an output tile
// is 256 x 256 and belongs to a cluster of two CTAs on two SMs.  Each CTA loads
// half of the A rows (its 128 output rows) and half of the B columns (128) of
// every K block into its own shared memory; one thread of the first CTA (the
// leader) issues tcgen05.mma.cta_group::2 with M = 256, which reads both CTAs'
// halves and leaves each CTA's 128 x 256 fp32 rows in that CTA's tensor memory.
// Per output element each SM therefore stages and feeds the tensor core two
// thirds of the operand bytes of the one-CTA tile (32 KB instead of 48 KB per
// 64-deep K block), which is what bounds a 128 x 256 tile on one SM.
//
// Roles (320 threads in each CTA):
//   warp 0   producer.  Leader: takes tile indices from the global counter and
//            hands each to both CTAs through their shared-memory tile rings;
//            both CTAs TMA-load their own halves.  The leader's stage barrier
//            counts its own bytes, the peer's bytes (its loads signal the
//            leader's barrier) and one arrival of the peer.
//   warp 1   leader: TMEM and the MMA issuer; the MMAs' commits free the stage
//            in both CTAs and hand finished accumulators to both epilogues.
//            Peer: only allocates and frees its half of the tensor memory.
//   warps 2-9  epilogue in both CTAs, each on its own 128 rows; the leader may
//            reuse an accumulator once all 16 epilogue warps have drained it.
// Variable K (wgrad): the last K block of an expert would reach into the next
// expert's rows.  It is loaded through row-window tensor maps whose window ends
// at the expert's last row, so the rows past it arrive as zeros; only an expert
// that ends before packed row 64 (no window fits) is zeroed by the leader's MMA
// warp in both CTAs' shared memory.  Every wait is bounded (LRMOE_ST_TIMEOUT, then a clean exit through
// a cluster barrier, so that neither CTA leaves while the other can still
// touch its shared memory).  No TMA multicast.
#include <type_traits>

#include "gemm_common.cuh"

namespace lrmoe {
namespace {

constexpr int kPairM = 2 * BM;               // MMA M of the pair
constexpr int kHalfN = kBNT / 2;             // B columns loaded by each CTA
constexpr int kPairABytes = BM * BK * 2;     // 16 KB: this CTA's 128 A rows of a K block
constexpr int kPairBBytes = kHalfN * BK * 2; // 16 KB: this CTA's 128 B columns
constexpr int kPairStage = kPairABytes + kPairBBytes;
// warps that read a tile-ring slot: the leader's MMA warp, the peer's producer, and
// the epilogue warps of both CTAs
__host__ __device__ constexpr int pair_consumers() { return 2 * (1 + kEpiWarps); }

// Launch counter of the pair kernels (picks the scheduling slot).
std::atomic<unsigned int> g_launches{0};

template <int STAGES, int OUTBUFS>
struct PairLayout {
  static constexpr int kTilesBytes = STAGES * kPairStage;
  static constexpr int kOutBufBytes = 32 * 32 * 4;
  static constexpr int kOutOff = kTilesBytes;
  static constexpr int kOutBytes = kEpiWarps * OUTBUFS * kOutBufBytes;
  static constexpr int kBarOff = kOutOff + kOutBytes;
  // per stage: full (leader), empty; tfull[2], tempty[2], mma_done; per ring
  // slot: full, empty
  static constexpr int kNumBars = 2 * STAGES + 5 + 2 * kRing;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag, tile ring
  static constexpr int kTableOff = kMiscOff + 16 + 4 * kRing;
  __host__ __device__ static constexpr int table_ints(int E) { return 3 * (E + 1) + 33; }
  __host__ __device__ static constexpr int alloc(int E) {
    return kTableOff + table_ints(E) * 4 + 1024;
  }
};

struct PairTile {
  int e;        // expert
  int row0;     // dgrad: first packed row of the 256-row tile; wgrad: the expert's first row
  int row_end;  // end of the expert's rows
  int m0, n0;   // wgrad: first output row (feature) of the pair tile; both: first column
  int nk;       // K blocks
  int narrow;   // at most 128 output columns left: an N = 128 MMA, 64 B columns per CTA
};

template <bool WG>
__device__ __forceinline__ PairTile decode_pair(int t, const GemmParams& p, const int* offs,
                                                const int* tab_d, const int* tab_w,
                                                const TileCounts& tc) {
  PairTile ti;
  if constexpr (WG) {
    const int per_e = tc.mt_w * tc.nt_w;
    const int oi = t / per_e, local = t - oi * per_e;
    ti.e = tab_w[oi];
    ti.m0 = (local / tc.nt_w) * kPairM;
    ti.n0 = (local % tc.nt_w) * kBNT;
    ti.row0 = offs[ti.e];
    ti.row_end = offs[ti.e + 1];
    ti.nk = (ti.row_end - ti.row0 + BK - 1) / BK;
    ti.narrow = p.N2 - ti.n0 <= kHalfN;
  } else {
    const int e = find_group(tab_d, p.E, t);
    const int local = t - tab_d[e];
    ti.e = e;
    ti.m0 = 0;
    ti.n0 = (local % tc.nt_d) * kBNT;
    ti.row0 = dgrad_tile_row0(offs[e], offs[e + 1] - offs[e], kPairM, p.part, local / tc.nt_d);
    ti.row_end = offs[e + 1];
    ti.nk = (p.Kd + BK - 1) / BK;
    // dgrad keeps 256-column MMAs on its last column tile too (the columns past Nd
    // load as zeros and are not stored): with the narrow form compiled in, both
    // dgrad launches of a T=16384, E=128, H=4096, I=1408 layer measured 3-10%
    // slower, the one without any narrow tile included
    ti.narrow = 0;
  }
  return ti;
}

// Zero rows [valid, valid + rows_bad) of the four 64-column chunks (A: two, B: two;
// 128-byte rows) of one stage in both CTAs of the pair, through cluster addresses
// (own: rank 0, peer: rank 1).  One warp.
__device__ __forceinline__ void zero_rows_both(uint32_t own, uint32_t peer, int valid,
                                               int rows_bad, int lane) {
  const int per_chunk = rows_bad * 8;  // 16-byte pieces per chunk
  for (int i = lane; i < 8 * per_chunk; i += 32) {
    const int c = i / per_chunk, rem = i - c * per_chunk;  // c: CTA * 4 + chunk
    const uint32_t off =
        (uint32_t)((c & 3) * 8192 + (valid + (rem >> 3)) * 128 + (rem & 7) * 16);
    st_cluster_zero16((c < 4 ? own : peer) + off);
  }
}

// MODE: kDgradStore, kDgradSwiglu or kWgrad.  STAGES = ring depth; OUTBUFS =
// fp32 staging buffers per epilogue warp (wgrad).
template <int MODE, int STAGES, int OUTBUFS>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_pair(
    const __grid_constant__ CUtensorMap tmA /* dgrad rows (K-major) / wgrad grad rows */,
    const __grid_constant__ CUtensorMap tmB /* dgrad W [E][K][N] / wgrad in rows */,
    const __grid_constant__ CUtensorMap tmOut /* wgrad dW [E][N1][N2] fp32 */,
    const __grid_constant__ CUtensorMap tmTA /* wgrad K-tail row windows over tmA's rows */,
    const __grid_constant__ CUtensorMap tmTB /* the same over tmB's rows */,
    const GemmParams p) {
  constexpr bool WG = MODE == kWgrad;
  constexpr bool SWIGLU = MODE == kDgradSwiglu;
  constexpr int BN = kBNT;
  using L = PairLayout<STAGES, OUTBUFS>;
  const int E = p.E;
  uint32_t* status = p.status;
  const uint64_t wlim = p.wait_ns ? p.wait_ns : kWaitLimitNs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;       // [2]
  uint64_t* tempty = bars + 2 * STAGES + 2;  // [2]
  uint64_t* mma_done = bars + 2 * STAGES + 4;
  uint64_t* ring_full = bars + 2 * STAGES + 5;           // [kRing]
  uint64_t* ring_empty = bars + 2 * STAGES + 5 + kRing;  // [kRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  volatile int* ring = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 16);  // [kRing]
  unsigned int* sched = g_sched[p.sched_slot];
  int* tab_w = reinterpret_cast<int*>(smem + L::kTableOff);
  int* tab_d = tab_w + (E + 1);
  int* scratch = tab_d + (E + 1);
  int* offs_s = scratch + 33;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 2);  // leader's arrive.expect_tx + one arrival of the peer
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * kEpiWarps);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], pair_consumers());
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if constexpr (WG) {
      tma_prefetch_desc(&tmTA);
      tma_prefetch_desc(&tmTB);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * BN);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers exist before either side arrives on the other's
  cluster_sync_all();
  pdl_wait();
  pdl_trigger();
  TileCounts tc{0, 0, 0, 0, 0, 0};
  if constexpr (WG) {
    tc.mt_w = (p.N1 + kPairM - 1) / kPairM;
    tc.nt_w = (p.N2 + BN - 1) / BN;
    build_wgrad_order(p.offsets, E, tab_w, tab_d);
    tc.tw = E * tc.mt_w * tc.nt_w;
  } else {
    tc.nt_d = (p.Nd + BN - 1) / BN;
    tc.td = build_dgrad_tiles(p.offsets, E, kPairM, tc.nt_d, tab_d, scratch, p.part);
  }
  tc.total = tc.td + tc.tw;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) offs_s[i] = p.offsets[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (offsets_invalid(offs_s, E, p.rows_cap, status)) tc.total = tc.td = tc.tw = 0;
  const uint32_t tmem_base = *tmem_slot;
  // cluster-window addresses of the leader's barriers that both CTAs arrive on
  const uint32_t lead_ring_empty = cluster_addr(ring_empty, 0);
  const uint32_t lead_tempty = cluster_addr(tempty, 0);
  const uint32_t lead_full = cluster_addr(full, 0);

  // Tile of the it-th round for this CTA's consumer warps (-1: no more tiles).
  auto next_tile = [&](int it) -> int {
    const int slot = it % kRing;
    // the leader's ring is written by its own producer (CTA scope); the peer's by
    // the leader's producer across the cluster
    const uint32_t par = (uint32_t)(it / kRing) & 1u;
    const bool ok = __all_sync(
        kFull, leader ? mbar_wait_bounded(&ring_full[slot], par, abort_flag, status, wlim)
                      : mbar_wait_bounded<true>(&ring_full[slot], par, abort_flag, status, wlim));
    const int t = ok ? ring[slot] : -1;
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(lead_ring_empty + 8u * slot);
    return t;
  };

  if (warp == 0) {
    // ---------------- producer ----------------
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0, armed_par = 0;  // leader: stages with loads issued, and their phase
    const uint32_t peer_ring = cluster_addr((const void*)ring, 1);
    const uint32_t peer_ring_full = cluster_addr(ring_full, 1);
    // Leader: claim a tile and hand it to both CTAs' consumers in ring slot it2 % kRing
    // (lane 0).  Tiles are claimed and published one ahead of the loads, so that the
    // peer knows its next tile before it finishes the current one.
    auto publish = [&](int it2) -> int {
      const int slot2 = it2 % kRing;
      int t2 = (int)atomicAdd(&sched[0], 1u);
      if (!mbar_wait_bounded<true>(&ring_empty[slot2], ((uint32_t)(it2 / kRing) & 1u) ^ 1u,
                                   abort_flag, status, wlim) ||
          t2 >= tc.total || *abort_flag)
        t2 = -1;
      ring[slot2] = t2;
      st_cluster_u32(peer_ring + 4u * slot2, (uint32_t)t2);
      mbar_arrive(&ring_full[slot2]);
      mbar_arrive_cluster(peer_ring_full + 8u * slot2);
      return t2;
    };
    int ahead = -1;  // leader: the tile published for the next round
    if (leader && lane == 0) ahead = publish(0);
    for (int it = 0;; ++it) {
      int t = -1;
      if (leader) {
        if (lane == 0) {
          t = ahead;
          if (t >= 0) ahead = publish(it + 1);
        }
        t = __shfl_sync(kFull, t, 0);
      } else {
        t = next_tile(it);
      }
      if (t < 0) break;
      const PairTile ti = decode_pair<WG>(t, p, offs_s, tab_d, tab_w, tc);
      // one K block: wait for its stage, then both CTAs' copies; the last block of a
      // wgrad tile may be a K tail (the loop over the other blocks carries no tail
      // logic at all)
      auto load_block = [&](int kb, auto last_c) -> bool {
        constexpr bool kLast = decltype(last_c)::value && WG;
        if (!__all_sync(kFull, mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, status,
                                                 wlim)))
          return false;
        if (p.stall && it == 0 && kb == 0) {  // diagnostic: this block never arrives
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          return true;
        }
        uint8_t* sa = smem + stage * kPairStage;
        uint8_t* sb = sa + kPairABytes;
        const int r = ti.row0 + kb * BK;
        // wgrad K-tail block (fewer than 64 of the expert's rows left): loaded through
        // the row-window maps, whose window ends at the expert's last row, so that
        // the rows past it land as zeros.  An expert that ends before packed row 64
        // has no such window: its tail block is loaded plainly and the MMA warp
        // zeroes the rows past the end (rare: only the first rows of the buffer).
        bool win = false;
        int tw = 0, te = 0;  // window coordinates
        if constexpr (kLast) {
          const int valid = ti.row_end - r;
          win = valid < BK && ti.row_end >= BK;
          tw = BK - valid;
          te = ti.row_end - BK;
        }
        const int a_c0 = WG ? ti.m0 + (int)rank * BM : kb * BK;  // A coordinates of this CTA
        const int a_c1 = WG ? r : ti.row0 + (int)rank * BM;
        // B columns of this CTA: 128 (two 64-column boxes), or 64 on a narrow tile
        const int b_col = ti.n0 + (int)rank * (ti.narrow ? 64 : kHalfN);
        const uint32_t cta_bytes = kPairABytes + (ti.narrow ? kPairBBytes / 2 : kPairBBytes);
        if (leader) {
          if (lane == 0) {
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            mbar_arrive_expect_tx(&full[stage], 2 * cta_bytes);
            if constexpr (WG) {
              if (win) {
                tma_load_3d(sa, &tmTA, &full[stage], a_c0, tw, te);
                tma_load_3d(sa + 8192, &tmTA, &full[stage], a_c0 + 64, tw, te);
                tma_load_3d(sb, &tmTB, &full[stage], b_col, tw, te);
                if (!ti.narrow) tma_load_3d(sb + 8192, &tmTB, &full[stage], b_col + 64, tw, te);
              } else {
                tma_load_2d(sa, &tmA, &full[stage], a_c0, a_c1);
                tma_load_2d(sa + 8192, &tmA, &full[stage], a_c0 + 64, a_c1);
                tma_load_2d(sb, &tmB, &full[stage], b_col, r);
                if (!ti.narrow) tma_load_2d(sb + 8192, &tmB, &full[stage], b_col + 64, r);
              }
            } else {
              tma_load_2d(sa, &tmA, &full[stage], a_c0, a_c1);
              tma_load_3d(sb, &tmB, &full[stage], b_col, kb * BK, ti.e);
              if (!ti.narrow) tma_load_3d(sb + 8192, &tmB, &full[stage], b_col + 64, kb * BK, ti.e);
            }
          }
        } else {
          if (lane == 0) {
            const uint32_t fb = lead_full + 8u * stage;
            if constexpr (WG) {
              if (win) {
                tma_load_3d_pair(sa, &tmTA, fb, a_c0, tw, te);
                tma_load_3d_pair(sa + 8192, &tmTA, fb, a_c0 + 64, tw, te);
                tma_load_3d_pair(sb, &tmTB, fb, b_col, tw, te);
                if (!ti.narrow) tma_load_3d_pair(sb + 8192, &tmTB, fb, b_col + 64, tw, te);
              } else {
                tma_load_2d_pair(sa, &tmA, fb, a_c0, a_c1);
                tma_load_2d_pair(sa + 8192, &tmA, fb, a_c0 + 64, a_c1);
                tma_load_2d_pair(sb, &tmB, fb, b_col, r);
                if (!ti.narrow) tma_load_2d_pair(sb + 8192, &tmB, fb, b_col + 64, r);
              }
            } else {
              tma_load_2d_pair(sa, &tmA, fb, a_c0, a_c1);
              tma_load_3d_pair(sb, &tmB, fb, b_col, kb * BK, ti.e);
              if (!ti.narrow) tma_load_3d_pair(sb + 8192, &tmB, fb, b_col + 64, kb * BK, ti.e);
            }
            mbar_arrive_cluster_relaxed(fb);  // the bytes themselves are counted by the barrier
          }
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      bool ok = true;
      if constexpr (WG) {  // the last block peeled off
        for (int kb = 0; kb + 1 < ti.nk; ++kb)
          if (!(ok = load_block(kb, std::false_type{}))) break;
        if (ok && ti.nk > 0) ok = load_block(ti.nk - 1, std::true_type{});
      } else {
        // dgrad: the same steps written inline in one loop (measured faster than the
        // block function for these instantiations)
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!__all_sync(kFull, mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, status,
                                                   wlim))) {
            ok = false;
            break;
          }
          if (p.stall && it == 0 && kb == 0) {  // diagnostic: this block never arrives
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          uint8_t* sa = smem + stage * kPairStage;
          uint8_t* sb = sa + kPairABytes;
          const int a_c1 = ti.row0 + (int)rank * BM;  // A rows of this CTA
          // B columns of this CTA: 128 (two 64-column boxes), or 64 on a narrow tile
          const int b_col = ti.n0 + (int)rank * (ti.narrow ? 64 : kHalfN);
          const uint32_t cta_bytes = kPairABytes + (ti.narrow ? kPairBBytes / 2 : kPairBBytes);
          if (leader) {
            if (lane == 0) {
              armed |= 1u << stage;
              armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
              mbar_arrive_expect_tx(&full[stage], 2 * cta_bytes);
              tma_load_2d(sa, &tmA, &full[stage], kb * BK, a_c1);
              tma_load_3d(sb, &tmB, &full[stage], b_col, kb * BK, ti.e);
              if (!ti.narrow) tma_load_3d(sb + 8192, &tmB, &full[stage], b_col + 64, kb * BK, ti.e);
            }
          } else {
            if (lane == 0) {
              const uint32_t fb = lead_full + 8u * stage;
              tma_load_2d_pair(sa, &tmA, fb, kb * BK, a_c1);
              tma_load_3d_pair(sb, &tmB, fb, b_col, kb * BK, ti.e);
              if (!ti.narrow) tma_load_3d_pair(sb + 8192, &tmB, fb, b_col + 64, kb * BK, ti.e);
              mbar_arrive_cluster_relaxed(fb);  // the bytes themselves are counted by the barrier
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) break;
    }
    // Let every load this pair started land before shared memory is released:
    // the leader's stage barriers count the peer's bytes too.
    if (leader && lane == 0)
      for (int i = 0; i < STAGES; ++i)
        if ((armed >> i) & 1u) mbar_wait_drain<true>(&full[i], (armed_par >> i) & 1u);
    __syncwarp();
  } else if (warp == 1) {
    if (leader) {
      // ---------------- MMA issuer (leader only) ----------------
      constexpr uint32_t idesc_full = idesc_bf16_f32(kPairM, BN, WG, true);
      constexpr uint32_t idesc_narrow = idesc_bf16_f32(kPairM, kHalfN, WG, true);
      const uint32_t peer_empty = cluster_addr(empty, 1);
      const uint32_t peer_tfull = cluster_addr(tfull, 1);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_iter = 0;
      for (int it = 0;; ++it) {
        const int t = next_tile(it);
        if (t < 0) break;
        const PairTile ti = decode_pair<WG>(t, p, offs_s, tab_d, tab_w, tc);
        if (ti.nk == 0) continue;
        const uint32_t b = acc_iter & 1u, bphase = (acc_iter >> 1) & 1u;
        if (!__all_sync(kFull, mbar_wait_bounded(&tempty[b], bphase ^ 1u, abort_flag, status,
                                                 wlim)))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        // one K block: wait for both CTAs' copies and issue its MMAs; the last block of
        // a wgrad tile may be a K tail (the loop over the other blocks carries no tail
        // logic at all).  Every block's data is counted in transaction bytes; an early
        // K-tail block (see the producer) is zeroed here, after a wait at cluster scope
        // so that the peer's copy is ordered before those stores.
        auto mma_block = [&](int kb, auto last_c) -> bool {
          constexpr bool kLast = decltype(last_c)::value && WG;
          int valid = BK;
          bool early = false;
          if constexpr (kLast) {
            valid = ti.row_end - (ti.row0 + kb * BK);
            early = valid < BK && ti.row_end < BK;
          }
          const bool landed =
              early ? mbar_wait_bounded<true>(&full[stage], phase, abort_flag, status, wlim)
                    : mbar_wait_bounded(&full[stage], phase, abort_flag, status, wlim);
          if (!__all_sync(kFull, landed)) return false;
          tc_fence_after();
          uint8_t* sa = smem + stage * kPairStage;
          uint8_t* sb = sa + kPairABytes;
          int nkk = BK / UK;
          if constexpr (kLast) {
            // K-tail block: only the 16-row steps that hold the expert's rows (the
            // rest of the last step is zero)
            if (valid < BK) nkk = (valid + UK - 1) / UK;
            if (early && nkk * UK > valid) {
              zero_rows_both(cluster_addr(sa, 0), cluster_addr(sa, 1), valid, nkk * UK - valid,
                             lane);
              fence_proxy_async_cluster();
              __syncwarp();
            }
          }
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(sa), b_addr = smem_u32(sb);
            const uint32_t idesc = ti.narrow ? idesc_narrow : idesc_full;
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk) {
              if (kLast && kk >= nkk) break;
              const uint64_t adesc = WG ? smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                        : smem_desc_sw128(a_addr + kk * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, 8192, 1024);
              tc_mma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            // the stage is free in both CTAs once these MMAs have read it
            tc_commit_pair(smem_u32(&empty[stage]));
            tc_commit_pair(peer_empty + 8u * stage);
          }
          __syncwarp();
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          return true;
        };
        bool ok = true;
        if constexpr (WG) {  // the last block peeled off
          for (int kb = 0; kb + 1 < ti.nk; ++kb)
            if (!(ok = mma_block(kb, std::false_type{}))) break;
          if (ok) ok = mma_block(ti.nk - 1, std::true_type{});
        } else {
          // dgrad: the same steps written inline in one loop (measured faster than the
          // block function for these instantiations)
          for (int kb = 0; kb < ti.nk; ++kb) {
            // every block's data (both CTAs' halves) is counted in transaction bytes
            if (!__all_sync(kFull,
                            mbar_wait_bounded(&full[stage], phase, abort_flag, status, wlim))) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t* sa = smem + stage * kPairStage;
            uint8_t* sb = sa + kPairABytes;
            if (lane == 0) {
              const uint32_t a_addr = smem_u32(sa), b_addr = smem_u32(sb);
#pragma unroll
              for (int kk = 0; kk < BK / UK; ++kk) {
                const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, 8192, 1024);
                tc_mma_f16_pair(d_tmem, adesc, bdesc, ti.narrow ? idesc_narrow : idesc_full,
                                (kb | kk) != 0 ? 1u : 0u);
              }
              // the stage is free in both CTAs once these MMAs have read it
              tc_commit_pair(smem_u32(&empty[stage]));
              tc_commit_pair(peer_empty + 8u * stage);
            }
            __syncwarp();
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        if (lane == 0) {
          tc_commit_pair(smem_u32(&tfull[b]));
          tc_commit_pair(peer_tfull + 8u * b);
        }
        __syncwarp();
        ++acc_iter;
      }
      // every issued MMA has finished before tensor memory is released, also
      // when another role gave up a wait
      if (lane == 0) tc_commit_pair(smem_u32(mma_done));
      __syncwarp();
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    constexpr int kCW = BN / 64;  // 32-column chunks per warp
    const int ew = warp - 2;
    const int q = warp & 3;
    const int cbase = (ew >> 2) * kCW;
    const int row_in_tile = (int)rank * BM + q * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    uint32_t acc_iter = 0;
    uint8_t* obuf = smem + L::kOutOff + ew * OUTBUFS * L::kOutBufBytes;
    uint32_t obuf_iter = 0;
    uint32_t ra[32], rb[32];
    auto release_acc = [&](uint32_t b) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_tempty + 8u * b);
    };
    for (int it = 0;; ++it) {
      const int t = next_tile(it);
      if (t < 0) break;
      const PairTile ti = decode_pair<WG>(t, p, offs_s, tab_d, tab_w, tc);
      const bool zero_tile = WG && ti.nk == 0;
      if (zero_tile && p.accumulate) continue;  // adding zero changes nothing
      uint32_t b = 0;
      if (!zero_tile) {
        b = acc_iter & 1u;
        const uint32_t bphase = (acc_iter >> 1) & 1u;
        if (!__all_sync(kFull, mbar_wait_bounded(&tfull[b], bphase, abort_flag, status, wlim)))
          break;
        tc_fence_after();
        tmem_ld_32x32b_x32(lane_base + b * BN + cbase * 32, ra);
        tmem_wait_ld();
        reg_fence(ra);
        if (kCW == 1) release_acc(b);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) ra[i] = rb[i] = 0u;
      }
      const int row = ti.row0 + row_in_tile;  // dgrad output row
      bool row_ok = !WG && row < ti.row_end;
      int gu_row = row;
      if constexpr (SWIGLU) {
        if (row_ok && p.perm != nullptr) {
          gu_row = p.perm[row];
          if (gu_row < 0 || gu_row >= p.gu_rows) {
            raise_status(status, LRMOE_ST_BAD_INDEX);
            row_ok = false;
          }
        }
      }
      uint4 ga[4], ua[4], gb[4], ub[4];
      if constexpr (SWIGLU) {
        if (row_ok) load_gu(ga, ua, p.Gp, p.Up, gu_row, ti.n0 + cbase * 32, p.Nd);
      }
      auto step = [&](uint32_t (&cur)[32], uint32_t (&nxt)[32], uint4 (&gc)[4], uint4 (&uc)[4],
                      uint4 (&gn)[4], uint4 (&un)[4], int i) {
        const int ch = cbase + i;
        const bool more = i + 1 < kCW;
        if (more && !zero_tile) tmem_ld_32x32b_x32(lane_base + b * BN + (ch + 1) * 32, nxt);
        const int nb = ti.n0 + ch * 32;
        if constexpr (WG) {
          const int mrow = ti.m0 + (int)rank * BM + q * 32;
          if (mrow < p.N1 && nb < p.N2) {
            uint8_t* buf = obuf + (obuf_iter % OUTBUFS) * L::kOutBufBytes;
            ++obuf_iter;
            if (lane == 0) bulk_wait_group_read<OUTBUFS - 1>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int slot = j ^ (lane & 7);
              *reinterpret_cast<uint4*>(buf + lane * 128 + slot * 16) =
                  make_uint4(cur[4 * j], cur[4 * j + 1], cur[4 * j + 2], cur[4 * j + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (p.accumulate)
                tma_reduce_add_3d(&tmOut, buf, nb, mrow, ti.e);
              else
                tma_store_3d(&tmOut, buf, nb, mrow, ti.e);
              bulk_commit_group();
            }
          }
        } else if constexpr (SWIGLU) {
          if (more && row_ok) load_gu(gn, un, p.Gp, p.Up, gu_row, nb + 32, p.Nd);
          if (row_ok) {
            uint16_t* og = static_cast<uint16_t*>(p.out_d) + (size_t)row * 2 * p.Nd;
            epi_swiglu(cur, gc, uc, og, og + p.Nd, nb, p.Nd);
          }
        } else {
          if (row_ok)
            epi_store_bf16(cur, static_cast<uint16_t*>(p.out_d) + (size_t)row * p.Nd, nb, p.Nd);
        }
        if (more && !zero_tile) {
          tmem_wait_ld();
          reg_fence(nxt);
          if (i + 2 == kCW) release_acc(b);  // last chunk is in registers
        }
      };
#pragma unroll
      for (int i = 0; i < kCW; ++i) {
        if (i & 1)
          step(rb, ra, gb, ub, ga, ua, i);
        else
          step(ra, rb, ga, ua, gb, ub, i);
      }
      if (!zero_tile) ++acc_iter;
    }
    if constexpr (WG) {
      if (lane == 0) bulk_wait_group<0>();  // shared memory must outlive the bulk stores
      __syncwarp();
    }
  }
  // Neither CTA leaves (or frees tensor memory) while the other may still read
  // its shared memory or arrive on its barriers.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 2 * BN);
  if (leader && threadIdx.x == 0) {
    // every tile request of this pair is done: the last pair out zeroes the slot
    __threadfence();
    if (atomicAdd(&sched[1], 1u) == gridDim.x / 2 - 1) {
      sched[0] = 0;
      sched[1] = 0;
      __threadfence();
    }
  }
}

template <int MODE, int S, int OB>
cudaError_t launch_pair_variant(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& out,
                                const CUtensorMap& ta, const CUtensorMap& tb, GemmParams prm,
                                cudaStream_t s, long long tiles) {
  using L = PairLayout<S, OB>;
  const int smem = L::alloc(prm.E);
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  auto kern = grouped_gemm_pair<MODE, S, OB>;
  // set on every launch (host-side only): a cached flag would go stale when the
  // device's context is reset
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // as many pairs as can be resident at once (a persistent grid), at most one per tile
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
    cudaGetLastError();  // clear a failed query
    clusters = num_sms() / 2;
  }
  if (tiles < clusters) clusters = (int)(tiles > 0 ? tiles : 1);
  cfg.gridDim = dim3(2 * clusters);
  cfg.numAttrs = 2;
  prm.sched_slot = (int)(g_launches.fetch_add(1u) % kSchedSlots);
  return cudaLaunchKernelEx(&cfg, kern, a, b, out, ta, tb, prm);
}

}  // namespace

// dgrad on pairs of SMs: D[R_e] = rows[R_e] (K-major) . W[e] (N-major); store or
// SwiGLU-backward epilogue (g, u at row perm[r] when perm is given).
cudaError_t launch_dgrad_pair(const void* rows, int rows_cap, const void* W,
                              const int32_t* offsets, int E, int K, int N, lrmoe_epilogue epi,
                              const void* Gp, const void* Up, void* out, uint32_t* status,
                              cudaStream_t s, const char** why, const int32_t* perm,
                              int gu_rows, int part) {
  CUtensorMap a, b;
  if (!make_map_2d(&a, rows, (uint64_t)rows_cap, (uint64_t)K, 64, 128) ||
      !make_map_3d(&b, W, (uint64_t)E, (uint64_t)K, (uint64_t)N)) {
    *why = "cuTensorMapEncodeTiled failed for a dgrad operand";
    return cudaErrorInvalidValue;
  }
  GemmParams prm{offsets, E, K, N, 0, 0, static_cast<const uint16_t*>(Gp),
                 static_cast<const uint16_t*>(Up), perm, gu_rows, out, 0, nullptr, 1, 0, status, 0,
                 0, 0, part, 0};
  prm.rows_cap = rows_cap;
  // an upper bound of the tile count (the real one is built on the device)
  const long long tiles =
      ((long long)rows_cap / kPairM + E) * ((N + kBNT - 1) / kBNT);
  if (epi == LRMOE_EPI_SWIGLU_BWD)
    return launch_pair_variant<kDgradSwiglu, 6, 0>(a, b, a, a, a, prm, s, tiles);
  return launch_pair_variant<kDgradStore, 6, 0>(a, b, a, a, a, prm, s, tiles);
}

// Diagnostic: the dgrad (store epilogue) with the first K block withheld and every
// wait limited to wait_ns; must end with LRMOE_ST_TIMEOUT and a usable context.
cudaError_t launch_dgrad_stall_pair(const void* rows, int rows_cap, const void* W,
                                    const int32_t* offsets, int E, int K, int N, void* out,
                                    unsigned long long wait_ns, uint32_t* status, cudaStream_t s) {
  CUtensorMap a, b;
  if (!make_map_2d(&a, rows, (uint64_t)rows_cap, (uint64_t)K, 64, 128) ||
      !make_map_3d(&b, W, (uint64_t)E, (uint64_t)K, (uint64_t)N))
    return cudaErrorInvalidValue;
  GemmParams prm{offsets, E, K, N, 0, 0, nullptr, nullptr, nullptr, 0, out, 0, nullptr, 1, 0,
                 status, 0, wait_ns, 1};
  prm.rows_cap = rows_cap;
  const long long tiles = ((long long)rows_cap / kPairM + E) * ((N + kBNT - 1) / kBNT);
  return launch_pair_variant<kDgradStore, 6, 0>(a, b, a, a, a, prm, s, tiles);
}

// wgrad on pairs of SMs: dW[e] = grad[R_e]^T . in[R_e] (fp32 out, stored or added).
cudaError_t launch_wgrad_pair(const void* grad_rows, const void* in_rows, int rows_cap,
                              const int32_t* offsets, int E, int N1, int N2, float* dW,
                              int accumulate, uint32_t* status, cudaStream_t s,
                              const char** why) {
  CUtensorMap a, b, out, ta, tb;
  if (!make_map_2d(&a, grad_rows, (uint64_t)rows_cap, (uint64_t)N1, 64, 64) ||
      !make_map_2d(&b, in_rows, (uint64_t)rows_cap, (uint64_t)N2, 64, 64) ||
      !make_map_rows_window(&ta, grad_rows, (uint64_t)rows_cap, (uint64_t)N1) ||
      !make_map_rows_window(&tb, in_rows, (uint64_t)rows_cap, (uint64_t)N2) ||
      !make_map_out_f32(&out, dW, (uint64_t)E, (uint64_t)N1, (uint64_t)N2)) {
    *why = "cuTensorMapEncodeTiled failed for a wgrad operand";
    return cudaErrorInvalidValue;
  }
  GemmParams prm{offsets, E, 0, 0, N1, N2, nullptr, nullptr, nullptr, 0, nullptr, accumulate,
                 nullptr, 1, 0, status, 0};
  prm.rows_cap = rows_cap;
  const long long tiles = (long long)E * ((N1 + kPairM - 1) / kPairM) * ((N2 + kBNT - 1) / kBNT);
  if (PairLayout<5, 1>::alloc(E) <= kSmemLimit)
    return launch_pair_variant<kWgrad, 5, 1>(a, b, out, ta, tb, prm, s, tiles);
  return launch_pair_variant<kWgrad, 4, 1>(a, b, out, ta, tb, prm, s, tiles);
}

}  // namespace lrmoe
