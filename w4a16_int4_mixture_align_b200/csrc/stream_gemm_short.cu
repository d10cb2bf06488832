// stream_gemm_short.cu -- the weight-streaming W4A16 grouped GEMM for K shorter than one
// stage (four 128-wide K tiles), e.g. K = 256, the down projection of the TP8 shard.
//
// An item then spans several adjacent 128-row tiles of its expert (adjacent in the blob),
// so that its one bulk copy still carries four tiles, and it is a single stage: it can
// never be split. Work is divided as whole items, round-robin over the CTAs:
//
//   warp 0        producer: takes the work items (routing block b, token chunk c, group of
//                 128-row tiles) two at a time, publishes both descriptors, then streams
//                 the two items' stages alternately, each stage ONE bulk copy of the
//                 item's tiles (codes + scales, 36 KiB: a bulk copy has a high fixed cost,
//                 so bytes per copy decide the streaming rate). The few routed activation
//                 rows are small and shared by every warp, so consumers read them straight
//                 from global memory through L1 (ld.global.nc) instead of staging them.
//   warps 1..8    consumer group 0 takes the first item of each pair, warps 9..16 group 1
//                 the second; a warp owns 16 physical rows of each tile. Codes go shared ->
//                 registers and dequantise to bf16 pairs (subtract 8, then scale) that are
//                 exactly the A fragments of mma.m16n8k16; tokens are N. After each tile's K
//                 the group runs its epilogue for that tile: SiLU(gate)*up (gate_up; gate
//                 and up rows are interleaved by the repack), the expert output (down) to the
//                 per-slot buffer y, or the plain output (grouped operators).
//
// (The stream-K division of stream_gemm.cu measured slower on these one-stage items, with
// the same bytes and about the same instructions: this kernel keeps the division that
// measured fastest here.)
//
// Every wait is an mbarrier wait bounded in time; on timeout the CTA raises
// CHORD_DEV_TIMEOUT, unwinds, and the producer waits (bounded) for its copies in flight.
#include "stream_common.cuh"

namespace chord {
namespace stream {
namespace {

constexpr int kDescRing = 32;

struct ItemDesc {
  int e, nt, pos0, end;     // end = 1 marks the end of the item sequence
  uint32_t s0;              // global index of the item's first stage
  int sstride;              // 2 when its stages alternate with the paired item's, else 1
  int pad[2];
  int f[kMaxTC];            // flat slot of each token column, -1 when padding
};

template <int TC>
struct Smem {
  static constexpr int kKTS = chord::stream::kKTS;
  static constexpr int kStageBytes = chord::stream::kStageBytes;
  static constexpr int kBudget = 200 * 1024;
  static constexpr int kFit = (kBudget - kDescRing * int(sizeof(ItemDesc)) - 1024) / kStageBytes;
  static constexpr int kStages = kFit > 12 ? 12 : kFit;
  static constexpr int kBytes = kStages * kStageBytes + kDescRing * int(sizeof(ItemDesc)) + 1024;
};

// MULTI: the item covers NTPI > 1 tiles of 128 rows (a K shorter than a stage, see NTPI)
template <int EPI, int TC, bool MULTI>
__global__ void __launch_bounds__(kThreads, 1) stream_gemm_kernel(StreamParams p) {
  using S = Smem<TC>;
  constexpr int NT8 = TC / 8;
  constexpr int NSTAGE = S::kStages;
  constexpr int KTS = S::kKTS;
  static_assert(NSTAGE >= 3 && NSTAGE < kDescRing, "stage count");
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stages = smem;
  ItemDesc* descs = reinterpret_cast<ItemDesc*>(smem + NSTAGE * S::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(descs) +
                                               kDescRing * sizeof(ItemDesc));
  uint64_t* full = bars;                        // [NSTAGE]
  uint64_t* empty = full + NSTAGE;              // [NSTAGE] the owning group's 8 warps
  uint64_t* dfull = empty + NSTAGE;             // [kDescRing]
  uint64_t* dempty = dfull + kDescRing;         // [kDescRing] the owning group's 8 warps
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    const BlobHeader* hd = reinterpret_cast<const BlobHeader*>(p.blob);
    if (hd->magic != kBlobMagic || hd->version != kBlobVersion || hd->layout != kLayoutTile128 ||
        int(hd->role) != p.role || hd->E != p.E || hd->N != p.N || hd->K != p.K) {
      abort_flag = 2;
      if (blockIdx.x == 0) atomicOr(p.status, CHORD_DEV_BLOB_MISMATCH);
    }
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    for (int s = 0; s < kDescRing; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dempty[s], 8);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (abort_flag) return;
  volatile int* abort_v = &abort_flag;

  const int KT = p.K / kTileK;
  const int NTILES = p.N / kTileN;
  // With a short K (KT < KTS) one tile's K would fill only part of a stage, and a bulk
  // copy's fixed cost makes small copies slow; an item then covers NTPI consecutive
  // 128-row tiles of its expert (adjacent in the blob), so one copy still carries up to
  // KTS tiles. NTPI divides NTILES.
  int NTPI = 1;
  if (MULTI && KT < KTS) {
    NTPI = KTS / KT;
    while (NTILES % NTPI) --NTPI;
  }
  const int KTI = KT * NTPI;                   // tiles per item
  const int KS = (KTI + KTS - 1) / KTS;        // stages per item
  const int NGRP = NTILES / NTPI;              // items per routing chunk
  const int cpb = (p.block_m + TC - 1) / TC;  // token chunks per routing block

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // Launched early (programmatic launch), the gate_up kernel may start while the routing
    // sort still runs: wait for it before reading the routing tensors. The down kernel's
    // producer reads only those tensors (complete before the gate_up kernel passed this
    // same wait) and the weights, so it starts streaming at once; its consumers wait for
    // the intermediate a.
    if (EPI != kDown) grid_dep_wait();
    const int ntp = routed_positions(p.ntp, p.block_m, p.cap, p.status);
    const int64_t nblocks = ntp / p.block_m;
    const int64_t items = nblocks * cpb * NGRP;
    const uint64_t pol_w = policy_evict_first();
    uint32_t stage = 0;      // global stage counter
    uint32_t nitem = 0;      // published descriptors
    bool ok = true;
    // routing metadata of item w: its expert and this lane's flat slot (lane < TC). The
    // loads run kLook items ahead (a small register queue) so their latency overlaps
    // the streaming of earlier items instead of stalling at every item boundary.
    constexpr int kLook = 4;
    auto load_meta = [&](int64_t w, int& e, int& pos0, int& f) {
      e = -1;
      pos0 = 0;
      f = -1;
      if (w >= items) return;
      const int64_t bc = w / NGRP;
      const int64_t b = bc / cpb;
      const int c = int(bc % cpb);
      e = __ldg(p.expert_ids + b);
      pos0 = int(b * p.block_m) + c * TC;
      const int lim = int(b * p.block_m) + p.block_m;
      if (lane < TC && pos0 + lane < lim) f = __ldg(p.sorted_ids + pos0 + lane);
    };
    int qe[kLook], qpos[kLook], qf[kLook];
#pragma unroll
    for (int i = 0; i < kLook; ++i) load_meta(blockIdx.x + int64_t(i) * gridDim.x, qe[i], qpos[i], qf[i]);
    int64_t w_next = blockIdx.x;
    // the next item with at least one routed row, or false at the end
    auto pop_item = [&](int& e, int& nt, int& pos0, int& fval) -> bool {
      while (w_next < items) {
        const int64_t w = w_next;
        w_next += gridDim.x;
        e = qe[0];
        pos0 = qpos[0];
        fval = qf[0];
        nt = int(w % NGRP);
#pragma unroll
        for (int i = 0; i + 1 < kLook; ++i) {
          qe[i] = qe[i + 1];
          qpos[i] = qpos[i + 1];
          qf[i] = qf[i + 1];
        }
        load_meta(w + int64_t(kLook) * gridDim.x, qe[kLook - 1], qpos[kLook - 1], qf[kLook - 1]);
        if (!(fval >= 0 && fval < p.n_slots) || unsigned(e) >= unsigned(p.E)) fval = -1;
        if (__ballot_sync(0xffffffffu, fval >= 0) != 0) return true;  // something routed here
      }
      return false;
    };
    // publishes one descriptor (or an end marker) at index nitem
    auto publish = [&](int e, int nt, int pos0, int fval, bool end, uint32_t s0, int sstride) -> bool {
      const uint32_t ds = nitem % kDescRing;
      if (nitem >= kDescRing &&
          !mbar_wait(&dempty[ds], ((nitem / kDescRing) - 1) & 1, abort_v, p.status))
        return false;
      ItemDesc* d = &descs[ds];
      if (lane < TC) d->f[lane] = fval;
      if (lane == 0) {
        d->e = e; d->nt = nt; d->pos0 = pos0; d->end = end ? 1 : 0; d->s0 = s0; d->sstride = sstride;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dfull[ds]);
      ++nitem;
      return true;
    };
    // streams stage ks of the item on expert e, tile nt: one bulk copy of up to KTS tiles
    auto stream_stage = [&](int e, int nt, int ks) -> bool {
      const uint32_t slot = stage % NSTAGE;
      if (stage >= uint32_t(NSTAGE) &&
          !mbar_wait(&empty[slot], ((stage / NSTAGE) - 1) & 1, abort_v, p.status))
        return false;
      const int kt0 = ks * KTS;
      const int ntl = min(KTS, KTI - kt0);
      if (lane == 0) {
        uint8_t* st = stages + slot * S::kStageBytes;
        const uint64_t tile0 = (uint64_t(e) * NTILES + uint64_t(nt) * NTPI) * KT;
        mbar_arrive_expect_tx(&full[slot], uint32_t(ntl) * kTileBytes);
        bulk_g2s_hint(st, p.tiles + (tile0 + kt0) * kTileBytes, uint32_t(ntl) * kTileBytes, &full[slot], pol_w);
      }
      ++stage;
      return true;
    };
    // items two at a time: group 0 takes the first, group 1 the second; their stages
    // alternate in the ring so both groups stream concurrently
    while (ok) {
      int ea, nta, pa, fa, eb, ntb, pb, fb;
      if (!pop_item(ea, nta, pa, fa)) break;
      const bool has_b = pop_item(eb, ntb, pb, fb);
      ok = publish(ea, nta, pa, fa, false, stage, has_b ? 2 : 1);
      if (ok && has_b) ok = publish(eb, ntb, pb, fb, false, stage + 1, 2);
      for (int ks = 0; ks < KS && ok; ++ks) {
        ok = stream_stage(ea, nta, ks);
        if (ok && has_b) ok = stream_stage(eb, ntb, ks);
      }
      if (!has_b) break;
    }
    // every stage is issued: the next kernel may launch and take SMs as CTAs here finish
    grid_dep_trigger();
    // end markers at two consecutive indices: one reaches each group
    if (ok) ok = publish(0, 0, 0, -1, true, 0, 1);
    if (ok) publish(0, 0, 0, -1, true, 0, 1);
    // drain: wait (bounded, ignoring the abort flag) for every copy still in flight
    if (lane == 0) {
      int dummy = 0;
      const uint32_t first = stage > uint32_t(NSTAGE) ? stage - NSTAGE : 0;
      for (uint32_t s = first; s < stage; ++s)
        mbar_wait(&full[s % NSTAGE], (s / NSTAGE) & 1, &dummy, p.status);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  if (EPI == kDown) grid_dep_wait();   // the intermediate a comes from the gate_up kernel
  const int cw = warp - 1;             // 0..15
  const int grp = cw >> 3;             // 0 or 1: the first or second item of each pair
  const int rb = cw & 7;               // 16-row block inside the tile
  const int g = lane >> 2, t = lane & 3;
  for (uint32_t it = grp;; it += 2) {
    const uint32_t ds = it % kDescRing;
    if (!mbar_wait(&dfull[ds], (it / kDescRing) & 1, abort_v, p.status)) return;
    const ItemDesc& d = descs[ds];
    if (d.end) return;
    // this lane's activation row of each 8-token tile (padding columns read row 0: their
    // results are discarded by the epilogue)
    const uint16_t* xrow0[NT8];
#pragma unroll
    for (int n8 = 0; n8 < NT8; ++n8) {
      const int f = d.f[n8 * 8 + g];
      const int64_t row = f < 0 ? 0
                          : (EPI == kGateUp ? int64_t(f / p.topk)
                                            : (EPI == kPlain ? int64_t(f) : int64_t(d.pos0 + n8 * 8 + g)));
      xrow0[n8] = p.act + row * p.act_ld;
    }
    // independent accumulator chains per 8-token tile so consecutive MMAs overlap
    constexpr int NSET = NT8 >= 4 ? 1 : (4 / NT8);
    float acc[NT8][NSET][4];
#pragma unroll
    for (int i = 0; i < NT8; ++i)
#pragma unroll
      for (int q = 0; q < NSET; ++q) acc[i][q][0] = acc[i][q][1] = acc[i][q][2] = acc[i][q][3] = 0.f;

    // this lane's 8 K of each row
    const uint16_t* xrow[NT8];
#pragma unroll
    for (int n8 = 0; n8 < NT8; ++n8) xrow[n8] = xrow0[n8] + 8 * t;

    // ---- epilogue of 128-row tile `ntile` (the item's last, or with a short K each of its
    // NTPI tiles in turn, leaving the accumulators zeroed for the next)
    auto epilogue = [&](int ntile) {
      float accs[NT8][4];
#pragma unroll
      for (int i = 0; i < NT8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v = 0.f;
#pragma unroll
          for (int q = 0; q < NSET; ++q) {
            v += acc[i][q][c];
            if (MULTI) acc[i][q][c] = 0.f;
          }
          accs[i][c] = v;
        }
      if (EPI == kGateUp) {
        const int i_col = ntile * (kTileN / 2) + rb * 8 + g;  // intermediate column
#pragma unroll
        for (int n8 = 0; n8 < NT8; ++n8) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int col = n8 * 8 + 2 * t + q;
            if (d.f[col] >= 0) {
              const float v = silu_mul(accs[n8][q], accs[n8][2 + q]);
              p.a_out[int64_t(d.pos0 + col) * p.I + i_col] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
          }
        }
      } else if (EPI == kPlain) {
        const int n0 = ntile * kTileN + rb * 16 + g;
#pragma unroll
        for (int n8 = 0; n8 < NT8; ++n8) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int f = d.f[n8 * 8 + 2 * t + q];
            if (f >= 0) {
              uint16_t* orow = p.out + int64_t(f) * p.N;
              orow[n0] = __bfloat16_as_ushort(__float2bfloat16_rn(accs[n8][q]));
              orow[n0 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(accs[n8][2 + q]));
            }
          }
        }
      } else {
        const int n0 = ntile * kTileN + rb * 16 + g;
#pragma unroll
        for (int n8 = 0; n8 < NT8; ++n8) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int col = n8 * 8 + 2 * t + q;
            const int f = d.f[col];
            if (f >= 0) {
              float* yr = p.y_out + int64_t(f) * p.H;
              yr[n0] = accs[n8][q];
              yr[n0 + 8] = accs[n8][2 + q];
            }
          }
        }
      }
    };

    const uint32_t s0 = d.s0;
    const int sstride = d.sstride;
    int kt = 0, sub = 0;  // MULTI: K tile inside the current 128-row tile, and that tile's index
    for (int ks = 0; ks < KS; ++ks) {
      const uint32_t s = s0 + uint32_t(ks * sstride);
      const uint32_t slot = s % NSTAGE;
      if (!mbar_wait(&full[slot], (s / NSTAGE) & 1, abort_v, p.status)) return;
      const int ntl = min(KTS, KTI - ks * KTS);
      // plain shared loads (ordered after the wait by its memory clobber) so the compiler
      // can schedule them ahead of the dequantisation and the MMAs
      const uint8_t* stg = stages + slot * S::kStageBytes;
      // software-pipelined over the stage's tiles: tile i + 1's codes are loaded from shared
      // memory before tile i is dequantised, so their latency overlaps the math
      TileCodes cur = load_tile_codes(stg, 0, rb, lane);
      for (int i = 0; i < ntl; ++i) {
        TileCodes nxt = cur;
        if (i + 1 < ntl) nxt = load_tile_codes(stg, i + 1, rb, lane);
        uint4 xv[4][NT8];
        load_tile_x<NT8>(xv, xrow, (MULTI ? kt : ks * KTS + i) * kTileK);
        consume_tile<NT8, NSET>(cur, xv, acc, (i & 1) * 2);
        cur = nxt;
        if (MULTI && ++kt == KT) {
          kt = 0;
          if (++sub < NTPI) epilogue(d.nt * NTPI + sub - 1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    epilogue(d.nt * NTPI + NTPI - 1);
    __syncwarp();
    if (lane == 0) mbar_arrive(&dempty[ds]);
  }
}

template <int EPI, int TC, bool MULTI>
cudaError_t launch_one(const StreamParams& p, int grid, bool pdl, cudaStream_t stream) {
  auto kern = stream_gemm_kernel<EPI, TC, MULTI>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<TC>::kBytes);
  if (err != cudaSuccess) return err;
  err = launch_pdl(pdl, kern, dim3(grid), dim3(kThreads), size_t(Smem<TC>::kBytes), stream, p);
  count_launches(1);
  return err != cudaSuccess ? err : cudaGetLastError();
}

template <int EPI, bool MULTI>
cudaError_t launch_tc_m(const StreamParams& p, int tc, int grid, bool pdl, cudaStream_t stream) {
  switch (tc) {
    case 8: return launch_one<EPI, 8, MULTI>(p, grid, pdl, stream);
    case 16: return launch_one<EPI, 16, MULTI>(p, grid, pdl, stream);
    default: return launch_one<EPI, 32, MULTI>(p, grid, pdl, stream);
  }
}

}  // namespace

cudaError_t launch_stream_gemm_short(int epi, const StreamParams& p, int tc, int grid, bool pdl,
                                     cudaStream_t stream) {
  switch (epi) {
    case kGateUp: return launch_tc_m<kGateUp, true>(p, tc, grid, pdl, stream);
    case kDown: return launch_tc_m<kDown, true>(p, tc, grid, pdl, stream);
    default: return launch_tc_m<kPlain, true>(p, tc, grid, pdl, stream);
  }
}

}  // namespace stream
}  // namespace chord
