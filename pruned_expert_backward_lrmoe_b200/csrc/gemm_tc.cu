// a4 for bf16 storage: variable-size grouped GEMMs on the sm_100a tensor cores.
//
// "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE", bullet 5
// (German page, paragraph 4: "gruppierte GEMMs variabler Größe"): the expert
// gradients are computed as grouped GEMMs over the compacted per-expert blocks
// with no zero padding.
//
// One persistent, warp-specialised kernel serves both shapes:
//   dgrad (variable M): D[R_e, :] = rows[R_e] (m_e x K) . W[e] (K x N)
//          A = rows, K-major;   B = W[e], N-major;  epilogue STORE or SwiGLU-bwd
//   wgrad (variable K): D = grad[R_e]^T (N1 x m_e) . in[R_e] (m_e x N2)
//          A = grad, M-major;   B = in, N-major;    epilogue fp32 store / add
// Roles (320 threads): warp 0 issues TMA loads into a ring of shared-memory
// stages; warp 1 owns tensor memory and one lane issues tcgen05.mma (128 x BN
// x 16 per instruction, fp32 accumulators in TMEM, two accumulator buffers so
// that the epilogue of one tile overlaps the main loop of the next); warps 2-9
// drain TMEM with tcgen05.ld and store.  Group sizes are read on the device.
// In wgrad the last K block of an expert may reach into the next expert's
// rows: those rows are zeroed in shared memory before the MMAs read them.
// Every mbarrier wait is bounded (LRMOE_ST_TIMEOUT, then a clean exit).
#include <stdlib.h>

#include "gemm_common.cuh"

namespace lrmoe {
namespace {

// STAGES = ring depth; OUTBUFS = fp32 staging buffers per epilogue warp (wgrad).
template <int MODE, int STAGES, int OUTBUFS>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_tc(
    const __grid_constant__ CUtensorMap tmAd /* dgrad rows, K-major boxes */,
    const __grid_constant__ CUtensorMap tmBd /* dgrad W [E][K][N] */,
    const __grid_constant__ CUtensorMap tmAw /* wgrad grad rows, MN-major boxes */,
    const __grid_constant__ CUtensorMap tmBw /* wgrad in rows */,
    const __grid_constant__ CUtensorMap tmOut /* wgrad dW [E][N1][N2] fp32 */,
    const GemmParams p) {
  using Tr = Traits<MODE>;
  constexpr int BN = kBNT;
  using L = Layout<BN, STAGES, OUTBUFS>;
  const int E = p.E;
  uint32_t* status = p.status;
  const uint64_t wlim = p.wait_ns ? p.wait_ns : kWaitLimitNs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;      // [2]
  uint64_t* tempty = bars + 2 * STAGES + 2; // [2]
  uint64_t* mma_done = bars + 2 * STAGES + 4;
  uint64_t* ring_full = bars + 2 * STAGES + 5;            // [kRing]
  uint64_t* ring_empty = bars + 2 * STAGES + 5 + kRing;   // [kRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  volatile int* ring = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 16);  // [kRing]
  unsigned int* sched = g_sched[p.sched_slot];
  // tables: wgrad expert order [E+1]; dgrad tile starts [E+1] (first used as the
  // wgrad build's size scratch); scan scratch [33]; offsets[0..E]
  int* tab_w = reinterpret_cast<int*>(smem + L::kTableOff);
  int* tab_d = tab_w + (E + 1);
  int* scratch = tab_d + (E + 1);
  int* offs_s = scratch + 33;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      // gathered B: the TMA arrival plus one cp.async arrival per producer lane
      mbar_init(&full[i], Tr::kGatherB ? 33 : 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiThreads);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 1 + kEpiWarps);  // MMA warp + each epilogue warp
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if constexpr (Tr::kHasD) {
      tma_prefetch_desc(&tmAd);
      tma_prefetch_desc(&tmBd);
    }
    if constexpr (Tr::kHasW) {
      tma_prefetch_desc(&tmAw);
      tma_prefetch_desc(&tmBw);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  // everything above touches no global memory; from here on, earlier kernels' outputs
  // (a late-wait launch reads only outputs that were complete when it started, see
  // GemmParams::late_wait, and waits for its predecessor at the end instead)
  if (!p.late_wait) {
    pdl_wait();
    pdl_trigger();
  }
  // tile tables
  TileCounts tc{0, 0, 0, 0, 0, 0};
  if constexpr (Tr::kHasW) {
    tc.mt_w = (p.N1 + BM - 1) / BM;
    tc.nt_w = (p.N2 + BN - 1) / BN;
    build_wgrad_order(p.offsets, E, tab_w, tab_d);
    tc.tw = E * tc.mt_w * tc.nt_w;
  }
  if constexpr (Tr::kHasD) {
    tc.nt_d = (p.Nd + BN - 1) / BN;
    tc.td = build_dgrad_tiles(p.offsets, E, BM, tc.nt_d, tab_d, scratch, p.part);
  }
  tc.total = tc.td + tc.tw;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) offs_s[i] = p.offsets[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (offsets_invalid(offs_s, E, p.rows_cap, status)) tc.total = tc.td = tc.tw = 0;
  const uint32_t tmem_base = *tmem_slot;

  // Tile of the it-th round for the MMA and epilogue warps (-1: no more tiles).
  auto next_tile = [&](int it) -> int {
    const int slot = it % kRing;
    const bool ok = __all_sync(
        kFull, mbar_wait_bounded(&ring_full[slot], (uint32_t)(it / kRing) & 1u, abort_flag, status, wlim));
    const int t = ok ? ring[slot] : -1;
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring_empty[slot]);
    return t;
  };

  if (Tr::kGatherB && warp == 0) {
    // ---------------- producer with gathered B (whole warp) ----------------
    // lane 0 schedules tiles and loads A by TMA; all lanes gather B: 64 rows x 256
    // columns per stage as 16-byte cp.async pieces written where a 128-byte
    // swizzled TMA box would put them (row rr at rr * 128, piece c at c ^ (rr & 7))
    if constexpr (Tr::kGatherB) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;  // stages with a load issued, and its phase
      unsigned int next = 0;
      if (lane == 0) next = atomicAdd(&sched[0], 1u);
      const int piece = lane & 7;
      for (int it = 0;; ++it) {
        const int slot = it % kRing;
        int t = -1;
        if (lane == 0) {
          t = (int)next;
          if (!mbar_wait_bounded(&ring_empty[slot], ((uint32_t)(it / kRing) & 1u) ^ 1u,
                                 abort_flag, status, wlim) ||
              t >= tc.total || *abort_flag)
            t = -1;
          ring[slot] = t;
          mbar_arrive(&ring_full[slot]);
        }
        t = __shfl_sync(kFull, t, 0);
        if (t < 0) break;
        const TileInfo ti = decode_tile<MODE>(t, p, offs_s, tab_d, tab_w, tc);
        if (ti.nk == 0 && lane == 0) next = atomicAdd(&sched[0], 1u);
        bool ok = true;
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!__all_sync(kFull, mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, status, wlim))) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * L::kStageBytes;
          uint8_t* sb = sa + L::kABytes;
          const int r0 = ti.row0 + kb * BK;
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (lane == 0) {
            if (kb == ti.nk - 1) next = atomicAdd(&sched[0], 1u);
            mbar_arrive_expect_tx(&full[stage], L::kABytes);
            tma_load_2d(sa, &tmAw, &full[stage], ti.m0, r0);
            tma_load_2d(sa + 8192, &tmAw, &full[stage], ti.m0 + 64, r0);
          }
          // perm of the block's 64 rows: lane l holds rows l and l + 32 (one round trip)
          int pv[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int r = r0 + lane + 32 * h;
            pv[h] = -1;
            if (r < ti.row_end) {
              const int pp = __ldg(p.perm + r);
              if (pp >= 0 && pp < p.gperm_max)
                pv[h] = pp / p.gdiv;
              else
                raise_status(status, LRMOE_ST_BAD_INDEX);
            }
          }
#pragma unroll
          for (int i = 0; i < BK / 4; ++i) {
            const int rr = (lane >> 3) + 4 * i;  // row inside the K block
            const long long srow = __shfl_sync(kFull, i < 8 ? pv[0] : pv[1], rr & 31);
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) {
              const int col = ti.n0 + c * 64 + piece * 8;
              const bool in = srow >= 0 && col < p.N2;
              const uint16_t* src = in ? p.gsrc + srow * p.N2 + col : p.gsrc;
              cp_async_16(sb + c * 8192 + rr * 128 + ((piece ^ (rr & 7)) * 16), src, in ? 16u : 0u);
            }
          }
          cp_async_arrive_noinc(&full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // Let every copy this warp started land before the CTA releases its shared
      // memory (they are all consumed already unless a wait gave up).
      cp_async_wait_all();
      if (lane == 0)
        for (int i = 0; i < STAGES; ++i)
          if ((armed >> i) & 1u) mbar_wait_drain(&full[i], (armed_par >> i) & 1u);
      __syncwarp();
    }
  } else if (warp == 0) {
    // ---------------- TMA producer (and tile scheduler) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;  // stages with a load issued, and its phase
      unsigned int next = atomicAdd(&sched[0], 1u);
      for (int it = 0;; ++it) {
        const int slot = it % kRing;
        int t = (int)next;
        if (!mbar_wait_bounded(&ring_empty[slot], ((uint32_t)(it / kRing) & 1u) ^ 1u, abort_flag, status, wlim) ||
            t >= tc.total || *abort_flag)
          t = -1;
        ring[slot] = t;
        mbar_arrive(&ring_full[slot]);
        if (t < 0) break;
        const TileInfo ti = decode_tile<MODE>(t, p, offs_s, tab_d, tab_w, tc);
        if (ti.nk == 0) next = atomicAdd(&sched[0], 1u);
        for (int kb = 0; kb < ti.nk; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, status, wlim)) break;
          // claim the following tile only now, a few K blocks before this one ends,
          // so that no CTA sits on a tile it cannot start soon
          if (kb == ti.nk - 1) next = atomicAdd(&sched[0], 1u);
          if (p.stall && it == 0 && kb == 0) {  // diagnostic: this block never arrives
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            continue;
          }
          uint8_t* sa = smem + stage * L::kStageBytes;
          uint8_t* sb = sa + L::kABytes;
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          if (ti.kind == 1) {
            if constexpr (Tr::kHasW) {
              const int r = ti.row0 + kb * BK;
              tma_load_2d(sa, &tmAw, &full[stage], ti.m0, r);
              tma_load_2d(sa + 8192, &tmAw, &full[stage], ti.m0 + 64, r);
#pragma unroll
              for (int c = 0; c < BN / 64; ++c)
                tma_load_2d(sb + c * 8192, &tmBw, &full[stage], ti.n0 + c * 64, r);
            }
          } else {
            if constexpr (Tr::kHasD) {
              tma_load_2d(sa, &tmAd, &full[stage], kb * BK, ti.row0);
#pragma unroll
              for (int c = 0; c < BN / 64; ++c)
                tma_load_3d(sb + c * 8192, &tmBd, &full[stage], ti.n0 + c * 64, kb * BK, ti.e);
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Let every TMA load this CTA started land before its shared memory is
      // released (after a normal run they have all been consumed already).
      for (int i = 0; i < STAGES; ++i)
        if ((armed >> i) & 1u) mbar_wait_drain(&full[i], (armed_par >> i) & 1u);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc_d = idesc_bf16_f32(BM, BN, false, true);  // A K-major
    constexpr uint32_t idesc_w = idesc_bf16_f32(BM, BN, true, true);   // A MN-major
    int stage = 0;
    uint32_t phase = 0;
    uint32_t acc_iter = 0;
    for (int it = 0;; ++it) {
      const int t = next_tile(it);
      if (t < 0) break;
      const TileInfo ti = decode_tile<MODE>(t, p, offs_s, tab_d, tab_w, tc);
      if (ti.nk == 0) continue;
      const bool wg = ti.kind == 1;
      const uint32_t b = acc_iter & 1u, bphase = (acc_iter >> 1) & 1u;
      if (!__all_sync(kFull, mbar_wait_bounded(&tempty[b], bphase ^ 1u, abort_flag, status, wlim)))
        break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + b * BN;
      bool ok = true;
      for (int kb = 0; kb < ti.nk; ++kb) {
        if (!__all_sync(kFull, mbar_wait_bounded(&full[stage], phase, abort_flag, status, wlim))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // gathered B was written by cp.async (generic proxy); the MMAs read it
        // through the async proxy
        if constexpr (Tr::kGatherB) fence_proxy_async_smem();
        uint8_t* sa = smem + stage * L::kStageBytes;
        uint8_t* sb = sa + L::kABytes;
        int nkk = BK / UK;  // MMAs of this K block
        if (Tr::kHasW && wg) {
          const int valid = ti.row_end - (ti.row0 + kb * BK);
          if (valid < BK) {
            // Last K block of the expert: only the 16-row groups that hold valid rows
            // are multiplied, and the rows of the last such group past the expert's
            // end (another expert's rows, or unwritten memory) are zeroed first.
            nkk = (valid + UK - 1) / UK;
            const int rows_bad = nkk * UK - valid;  // 0..15
            if (rows_bad > 0) {
              constexpr int nchunk = 2 + BN / 64;  // 64-wide column chunks of A and B
              const int per_chunk = rows_bad * 8;  // 16-byte pieces per chunk
              for (int i = lane; i < nchunk * per_chunk; i += 32) {
                const int ch = i / per_chunk;
                const int rem = i - ch * per_chunk;
                uint8_t* base = ch < 2 ? sa + ch * 8192 : sb + (ch - 2) * 8192;
                *reinterpret_cast<uint4*>(base + (valid + (rem >> 3)) * 128 + (rem & 7) * 16) =
                    make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async_smem();
              __syncwarp();
            }
          }
        }
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(sa), b_addr = smem_u32(sb);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            if (kk >= nkk) break;
            const uint64_t adesc = wg ? smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                      : smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, 8192, 1024);
            tc_mma_f16(d_tmem, adesc, bdesc, wg ? idesc_w : idesc_d, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&tfull[b]);
      __syncwarp();
      ++acc_iter;
    }
    // make sure every issued MMA has finished before tensor memory is released,
    // also when another role gave up a wait (the abort flag does not cut this short)
    if (lane == 0) tc_commit(mma_done);
    __syncwarp();
    mbar_wait_drain(mma_done, 0);
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    // Two warps per TMEM lane quarter q = warp % 4; warp half h owns the 32-column
    // chunks [h * kCW, (h + 1) * kCW) of the tile.  The next chunk's tcgen05.ld is
    // in flight while the current chunk is written out.
    constexpr int kCW = BN / 64;  // chunks per warp
    const int ew = warp - 2;
    const int q = warp & 3;
    const int cbase = (ew >> 2) * kCW;
    const int row_in_tile = q * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    uint32_t acc_iter = 0;
    // wgrad output staging: this warp's OUTBUFS 32 x 32 fp32 buffers (128-byte swizzled rows)
    uint8_t* obuf = smem + L::kOutOff + ew * OUTBUFS * L::kOutBufBytes;
    uint32_t obuf_iter = 0;
    uint32_t ra[32], rb[32];
    for (int it = 0;; ++it) {
      const int t = next_tile(it);
      if (t < 0) break;
      const TileInfo ti = decode_tile<MODE>(t, p, offs_s, tab_d, tab_w, tc);
      const bool wg = Tr::kHasW && ti.kind == 1;
      const bool zero_tile = wg && ti.nk == 0;
      if (zero_tile && p.accumulate) continue;  // adding zero changes nothing
      uint32_t b = 0;
      if (!zero_tile) {
        b = acc_iter & 1u;
        const uint32_t bphase = (acc_iter >> 1) & 1u;
        if (!__all_sync(kFull, mbar_wait_bounded(&tfull[b], bphase, abort_flag, status, wlim))) break;
        tc_fence_after();
        tmem_ld_32x32b_x32(lane_base + b * BN + cbase * 32, ra);
        tmem_wait_ld();
        reg_fence(ra);
        if (kCW == 1) {
          tc_fence_before();
          mbar_arrive(&tempty[b]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) ra[i] = rb[i] = 0u;
      }
      const int row = ti.row0 + row_in_tile;  // dgrad output row
      bool row_ok = !wg && row < ti.row_end;
      int gu_row = row;                        // SwiGLU: row of g, u
      if constexpr (Tr::kSwiglu) {
        if (row_ok && p.perm != nullptr) {
          gu_row = p.perm[row];
          if (gu_row < 0 || gu_row >= p.gu_rows) {
            raise_status(status, LRMOE_ST_BAD_INDEX);
            row_ok = false;
          }
        }
      }
      uint4 ga[4], ua[4], gb[4], ub[4];        // SwiGLU: saved g, u of the current / next chunk
      if constexpr (Tr::kSwiglu) {
        if (row_ok) load_gu(ga, ua, p.Gp, p.Up, gu_row, ti.n0 + cbase * 32, p.Nd);
      }
      auto step = [&](uint32_t (&cur)[32], uint32_t (&nxt)[32], uint4 (&gc)[4], uint4 (&uc)[4],
                      uint4 (&gn)[4], uint4 (&un)[4], int i) {
        const int ch = cbase + i;
        const bool more = i + 1 < kCW;
        if (more && !zero_tile) tmem_ld_32x32b_x32(lane_base + b * BN + (ch + 1) * 32, nxt);
        const int nb = ti.n0 + ch * 32;
        if (wg) {
          if constexpr (Tr::kHasW) {
            const int mrow = ti.m0 + q * 32;
            if (mrow < p.N1 && nb < p.N2) {
              uint8_t* buf = obuf + (obuf_iter % OUTBUFS) * L::kOutBufBytes;
              ++obuf_iter;
              // the store that last used `buf` has read it
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
          }
        } else if constexpr (Tr::kHasD) {
          if constexpr (Tr::kSwiglu) {
            if (more && row_ok) load_gu(gn, un, p.Gp, p.Up, gu_row, nb + 32, p.Nd);
            if (row_ok) {
              uint16_t* og = static_cast<uint16_t*>(p.out_d) + (size_t)row * 2 * p.Nd;
              epi_swiglu(cur, gc, uc, og, og + p.Nd, nb, p.Nd);
            }
          } else {
            if (row_ok)
              epi_store_bf16(cur, static_cast<uint16_t*>(p.out_d) + (size_t)row * p.Nd, nb, p.Nd);
          }
        }
        if (more && !zero_tile) {
          tmem_wait_ld();
          reg_fence(nxt);
          if (i + 2 == kCW) {  // last chunk is in registers: the accumulator is free
            tc_fence_before();
            mbar_arrive(&tempty[b]);
          }
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
  }
  if constexpr (Tr::kHasW) {
    // shared memory must outlive the bulk stores that read it
    if (warp >= 2 && lane == 0) bulk_wait_group<0>();  // every epilogue warp
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 2 * BN);
  if (threadIdx.x == 0) {
    // every tile request of this CTA is done: the last CTA out zeroes the slot
    __threadfence();
    if (atomicAdd(&sched[1], 1u) == gridDim.x - 1) {
      sched[0] = 0;
      sched[1] = 0;
      __threadfence();
    }
  }
  if (p.late_wait) {
    // this grid completes only after the kernel before it, so the next kernel in
    // the stream sees both kernels' rows
    pdl_wait();
    pdl_trigger();
  }
}


// Launch counter of all grouped-GEMM kernels (picks the scheduling slot).
std::atomic<unsigned int> g_launches{0};

struct Maps {
  CUtensorMap ad, bd, aw, bw, out;
};

// Launch one instantiation; the dynamic shared memory depends on E.
template <int MODE, int S, int OB>
cudaError_t launch_variant(const Maps& m, GemmParams prm, cudaStream_t s, int grid) {
  using L = Layout<kBNT, S, OB>;
  static_assert(L::alloc(kMaxExperts) <= kSmemLimit || OB == 1,
                "shared memory over the sm_100 per-block limit");
  const int smem = L::alloc(prm.E);
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  // Set on every launch (a host-side call, no device work): a cached "already
  // set" flag would go stale when the device's context is reset and recreated.
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_tc<MODE, S, OB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  if (err != cudaSuccess) return err;
  prm.sched_slot = (int)(g_launches.fetch_add(1u) % kSchedSlots);
  return launch_pdl(grouped_gemm_tc<MODE, S, OB>, dim3(grid), dim3(kThreads), (size_t)smem, s,
                    m.ad, m.bd, m.aw, m.bw, m.out, prm);
}

// dgrad K loops are long (K = H or 2I): 4 stages.  Launches with wgrad tiles
// stage their fp32 output in shared memory: 4 stages with one staging buffer
// per epilogue warp when that fits for this E (E <= ~140), else 3 stages with two.
template <int MODE>
cudaError_t launch_mode(const Maps& m, const GemmParams& prm, cudaStream_t s, int grid) {
  if constexpr (Traits<MODE>::kHasW) {
    if (Layout<kBNT, 4, 1>::alloc(prm.E) <= kSmemLimit)
      return launch_variant<MODE, 4, 1>(m, prm, s, grid);
    return launch_variant<MODE, 3, 2>(m, prm, s, grid);
  } else {
    return launch_variant<MODE, 4, 0>(m, prm, s, grid);
  }
}

bool dgrad_maps(Maps* m, const void* rows, int rows_cap, const void* W, int E, int K, int N) {
  return make_map_2d(&m->ad, rows, (uint64_t)rows_cap, (uint64_t)K, 64, 128) &&
         make_map_3d(&m->bd, W, (uint64_t)E, (uint64_t)K, (uint64_t)N);
}

bool wgrad_maps(Maps* m, const void* grad_rows, const void* in_rows, int rows_cap, int E, int N1,
                int N2, float* dW) {
  return make_map_2d(&m->aw, grad_rows, (uint64_t)rows_cap, (uint64_t)N1, 64, 64) &&
         make_map_2d(&m->bw, in_rows, (uint64_t)rows_cap, (uint64_t)N2, 64, 64) &&
         make_map_out_f32(&m->out, dW, (uint64_t)E, (uint64_t)N1, (uint64_t)N2);
}

}  // namespace

// The grouped dgrad and wgrad run on the two-SM tiles of gemm_pair.cu (a pair of
// SMs per 256 x 256 output tile).  LRMOE_GEMM_ONE_SM=1 in the environment selects
// the one-SM tiles of this file instead (128 x 256 per SM; faster for the dgrads
// of layers whose experts keep fewer than about 128 rows, where a 256-row tile
// is mostly empty).  Both compute the same result, bit for bit.
static bool one_sm_tiles() {
  static const bool v = [] {
    const char* e = getenv("LRMOE_GEMM_ONE_SM");
    return e != nullptr && e[0] == '1';
  }();
  return v;
}

// Default: each expert's rows in 256-row tiles on pairs of SMs (gemm_pair.cu), and
// a last tile of at most 128 rows on one SM in a second launch that runs as the
// first drains (a 256-row tile would leave half of its pair idle there).
cudaError_t launch_dgrad_tc(const void* rows, int rows_cap, const void* W,
                            const int32_t* offsets, int E, int K, int N, lrmoe_epilogue epi,
                            const void* Gp, const void* Up, void* out, uint32_t* status,
                            cudaStream_t s, const char** why, const int32_t* perm, int gu_rows) {
  const bool split = !one_sm_tiles();
  if (split) {
    const cudaError_t e = launch_dgrad_pair(rows, rows_cap, W, offsets, E, K, N, epi, Gp, Up, out,
                                            status, s, why, perm, gu_rows, kRowsPairs);
    if (e != cudaSuccess) return e;
  }
  Maps m;
  if (!dgrad_maps(&m, rows, rows_cap, W, E, K, N)) {
    *why = "cuTensorMapEncodeTiled failed for a dgrad operand";
    return cudaErrorInvalidValue;
  }
  m.aw = m.bw = m.out = m.ad;  // unused
  GemmParams prm{offsets, E, K, N, 0, 0, static_cast<const uint16_t*>(Gp),
                 static_cast<const uint16_t*>(Up), perm, gu_rows, out, 0, nullptr, 1, 0, status, 0,
                 0, 0, split ? kRowsTails : kRowsAll, split ? 1 : 0};
  prm.rows_cap = rows_cap;
  if (epi == LRMOE_EPI_SWIGLU_BWD) return launch_mode<kDgradSwiglu>(m, prm, s, num_sms());
  return launch_mode<kDgradStore>(m, prm, s, num_sms());
}

// Diagnostic: the one-SM dgrad (store epilogue) with the first K block withheld
// and every wait limited to wait_ns.
cudaError_t launch_dgrad_stall_tc(const void* rows, int rows_cap, const void* W,
                                  const int32_t* offsets, int E, int K, int N, void* out,
                                  unsigned long long wait_ns, uint32_t* status, cudaStream_t s) {
  Maps m;
  if (!dgrad_maps(&m, rows, rows_cap, W, E, K, N)) return cudaErrorInvalidValue;
  m.aw = m.bw = m.out = m.ad;  // unused
  GemmParams prm{offsets, E, K, N, 0, 0, nullptr, nullptr, nullptr, 0, out, 0, nullptr, 1, 0,
                 status, 0, wait_ns, 1};
  prm.rows_cap = rows_cap;
  return launch_mode<kDgradStore>(m, prm, s, num_sms());
}

cudaError_t launch_wgrad_tc(const void* grad_rows, const void* in_rows, int rows_cap,
                            const int32_t* offsets, int E, int N1, int N2, float* dW,
                            int accumulate, uint32_t* status, cudaStream_t s, const char** why) {
  if (!one_sm_tiles())
    return launch_wgrad_pair(grad_rows, in_rows, rows_cap, offsets, E, N1, N2, dW, accumulate,
                             status, s, why);
  Maps m;
  if (!wgrad_maps(&m, grad_rows, in_rows, rows_cap, E, N1, N2, dW)) {
    *why = "cuTensorMapEncodeTiled failed for a wgrad operand";
    return cudaErrorInvalidValue;
  }
  m.ad = m.bd = m.aw;  // unused
  const long long total = (long long)E * ((N1 + BM - 1) / BM) * ((N2 + kBNT - 1) / kBNT);
  int grid = num_sms();
  if (total < grid) grid = (int)total;
  GemmParams prm{offsets, E, 0, 0, N1, N2, nullptr, nullptr, nullptr, 0, nullptr, accumulate,
                 nullptr, 1, 0, status, 0};
  prm.rows_cap = rows_cap;
  return launch_mode<kWgrad>(m, prm, s, grid);
}

cudaError_t launch_wgrad_gather_tc(const void* grad_rows, int rows_cap, const int32_t* perm,
                                   const void* src, int src_div, int perm_max,
                                   const int32_t* offsets, int E, int N1, int N2, float* dW,
                                   int accumulate, uint32_t* status, cudaStream_t s,
                                   const char** why) {
  Maps m;
  if (!make_map_2d(&m.aw, grad_rows, (uint64_t)rows_cap, (uint64_t)N1, 64, 64) ||
      !make_map_out_f32(&m.out, dW, (uint64_t)E, (uint64_t)N1, (uint64_t)N2)) {
    *why = "cuTensorMapEncodeTiled failed for a wgrad operand";
    return cudaErrorInvalidValue;
  }
  m.ad = m.bd = m.bw = m.aw;  // unused
  const long long total = (long long)E * ((N1 + BM - 1) / BM) * ((N2 + kBNT - 1) / kBNT);
  int grid = num_sms();
  if (total < grid) grid = (int)total;
  GemmParams prm{offsets, E, 0, 0, N1, N2, nullptr, nullptr, perm, 0, nullptr, accumulate,
                 static_cast<const uint16_t*>(src), src_div, perm_max, status, 0};
  prm.rows_cap = rows_cap;
  return launch_mode<kWgradGather>(m, prm, s, grid);
}

cudaError_t launch_dgrad_wgrad_tc(const void* grad_rows, int rows_cap, const void* W,
                                  const int32_t* offsets, int E, int K, int N, lrmoe_epilogue epi,
                                  const void* Gp, const void* Up, void* out, const void* in_rows,
                                  int N2, float* dW, int accumulate, uint32_t* status,
                                  cudaStream_t s, const char** why) {
  Maps m;
  if (!dgrad_maps(&m, grad_rows, rows_cap, W, E, K, N) ||
      !wgrad_maps(&m, grad_rows, in_rows, rows_cap, E, K, N2, dW)) {
    *why = "cuTensorMapEncodeTiled failed for a fused dgrad/wgrad operand";
    return cudaErrorInvalidValue;
  }
  GemmParams prm{offsets, E, K, N, K, N2, static_cast<const uint16_t*>(Gp),
                 static_cast<const uint16_t*>(Up), nullptr, 0, out, accumulate, nullptr, 1, 0,
                 status, 0};
  prm.rows_cap = rows_cap;
  if (epi == LRMOE_EPI_SWIGLU_BWD) return launch_mode<kFusedSwiglu>(m, prm, s, num_sms());
  return launch_mode<kFusedStore>(m, prm, s, num_sms());
}

}  // namespace lrmoe
