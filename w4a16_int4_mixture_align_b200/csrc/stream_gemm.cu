// stream_gemm.cu -- weight-streaming W4A16 grouped GEMMs (few routed tokens per expert),
// for K of at least one stage (four 128-wide K tiles); shorter K runs the round-robin
// kernel of stream_gemm_short.cu.
//
// With few tokens routed to each expert the layer is bound by reading the packed
// weights once from HBM. The Chord blog's decode profile swaps the MMA operands so the
// dequantised weights fill the MMA-M slot and uses m16n8k16 ("H200 und Blackwell
// indexierter Decode"); the same operand orientation is used here, on sm_100a, with the
// weight tiles streamed by bulk asynchronous copies through a deep shared-memory ring.
// An item is (routing block b, token chunk c, 128-row tile nt) with KS stages of up to
// four K tiles; work is divided by stream-K ("H200 Prefill und TP8": Stream-K kept for
// the deep-K projections), so every consumer group streams the same number of stages:
//
//   warp 0        producer: owns the work ranges of the CTA's two consumer groups and
//                 issues ring stages for them strictly in turn (stage s for group s % 2),
//                 each stage ONE bulk copy of up to four consecutive 128-wide K tiles
//                 (codes + scales, 36 KiB: a bulk copy has a high fixed cost, so bytes per
//                 copy decide the streaming rate). For each piece of a group's range (the
//                 stages of one item inside it) it publishes a descriptor, with the
//                 routing metadata of the next piece already loaded. The few routed
//                 activation rows are small and shared by every warp, so consumers read
//                 them straight from global memory through L1 (ld.global.nc). (Copying each
//                 stage's activation slice into shared memory beside the weights, by the
//                 producer's lanes with cp.async, measured slower: the producer's time per
//                 stage is on the critical path.)
//   warps 1..8    consumer group 0, warps 9..16 group 1; a warp owns 16 physical rows and
//                 consumes every tile of its group's stages. Codes go shared -> registers
//                 and dequantise to bf16 pairs (subtract 8, then scale) that are exactly the
//                 A fragments of mma.m16n8k16; tokens are N. A piece that is a whole item
//                 runs the epilogue: SiLU(gate)*up (gate_up; gate and up rows are
//                 interleaved by the repack), the expert output (down) to the per-slot
//                 buffer y, which the combine weights and sums, or the plain output
//                 (grouped operators).
//
// Every wait is an mbarrier wait bounded in time; on timeout the CTA raises
// CHORD_DEV_TIMEOUT, unwinds, and the producer waits (bounded) for its copies in flight.
// The one wait on another CTA (a partial sum's flag) is bounded the same way and is
// never circular: a worker writes partials only for the first piece of its range and
// waits only in its last.
#include "stream_common.cuh"

namespace chord {
namespace stream {
namespace {

constexpr int kDescRingG = 8;  // descriptor ring of each consumer group

// How a piece (a run of stages of one item inside one worker's range) ends: the whole
// item (epilogue), the item's first stages (add the later parts' partials, then the
// epilogue) or a later part (store the partial and raise its flag).
enum PieceKind { kPieceFull = 0, kPieceOwner = 1, kPiecePart = 2 };

struct ItemDesc {
  int e, nt, pos0, end;     // end = 1 marks the end of the group's pieces
  int ks0, nks;             // the piece's stages of the item
  int kind;                 // PieceKind
  int v;                    // this worker (kPiecePart: its partial's slot)
  int vlast;                // kPieceOwner: partials come from workers v + 1 .. vlast
  int pad[3];
  int f[kMaxTC];            // flat slot of each token column, -1 when padding
};

template <int TC>
struct Smem {
  static constexpr int kFixed = 2 * kDescRingG * int(sizeof(ItemDesc)) + 1024;  // descriptors, barriers
  static constexpr int kFit = (kMaxDynSmem - kFixed) / kStageBytes;
  static constexpr int kStages = kFit > 12 ? 12 : kFit;
  static constexpr int kBytes = kStages * kStageBytes + kFixed;
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kBytes <= kMaxDynSmem, "shared memory");
};

// x / y for 0 <= x and 0 < y < 2^31, in 32-bit arithmetic whenever x fits (always, in
// practice): a 64-bit division is a long instruction sequence, and the producer divides
// unit and item indices several times per piece.
__device__ __forceinline__ int64_t div_fast(int64_t x, int y) {
  return x < (int64_t(1) << 31) ? int64_t(uint32_t(x) / uint32_t(y)) : x / y;
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <int EPI, int TC>
__global__ void __launch_bounds__(kThreads, 1) stream_gemm_kernel(StreamParams p) {
  using S = Smem<TC>;
  constexpr int NT8 = TC / 8;
  constexpr int NSTAGE = S::kStages;
  constexpr int KTS = kKTS;
  static_assert(NSTAGE >= 3, "stage count");
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stages = smem;
  ItemDesc* descs = reinterpret_cast<ItemDesc*>(smem + NSTAGE * kStageBytes);  // [2][kDescRingG]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(descs) +
                                               2 * kDescRingG * sizeof(ItemDesc));
  uint64_t* full = bars;                        // [NSTAGE]
  uint64_t* empty = full + NSTAGE;              // [NSTAGE] the owning group's 8 warps
  uint64_t* dfull = empty + NSTAGE;             // [2][kDescRingG]
  uint64_t* dempty = dfull + 2 * kDescRingG;    // [2][kDescRingG] the group's 8 warps
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
    for (int s = 0; s < 2 * kDescRingG; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dempty[s], 8);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (abort_flag) return;
  volatile int* abort_v = &abort_flag;

  const int KT = p.K / kTileK;                 // 128-wide K tiles (at least KTS here)
  const int NTILES = p.N / kTileN;             // 128-row tiles: items per routing chunk
  const int KS = (KT + KTS - 1) / KTS;         // stages per item
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
    const int64_t items = nblocks * cpb * NTILES;
    // Stream-K over P workers, one per consumer group (two per CTA): the (item, stage)
    // units, RU in all, form P equal contiguous ranges, so every group streams the same
    // number of stages (whole items per group leave a wave tail: with ~5 items per CTA,
    // 15% of the TP8 decode gate_up). An item cut by a range boundary is finished by the
    // worker holding its first stage, which reaches it last in its range; the workers
    // holding its other stages reach them first in theirs and leave FP32 partial sums.
    const int64_t P = 2 * int64_t(gridDim.x);
    const int64_t RU = items * KS;
    // (at most one worker per unit, so that every worker below PS holds at least one)
    const int64_t PS = min(P, RU > 0 ? RU : int64_t(1));
    auto range_start = [&](int64_t v) -> int64_t { return RU * v / PS; };
    auto worker_of = [&](int64_t u) -> int64_t {  // the worker whose range holds unit u
      int64_t v = u * PS / RU;
      while (v + 1 < PS && range_start(v + 1) <= u) ++v;
      while (v > 0 && range_start(v) > u) --v;
      return v;
    };
    const uint64_t pol_w = policy_evict_first();
    uint32_t stage = 0;  // global stage counter; stage s belongs to consumer group s % 2
    // routing metadata of item w: its expert, first position and this lane's flat slot
    // (lane < TC; -1 past the block). Only issues the loads: nothing here reads their
    // values, so a prefetch keeps them in flight until the piece starts (valid_slot).
    auto load_meta = [&](int64_t w, int& e, int& pos0, int& f) {
      const int64_t bc = div_fast(w, NTILES);
      const int64_t b = div_fast(bc, cpb);
      const int c = int(bc - b * cpb);
      e = __ldg(p.expert_ids + b);
      pos0 = int(b * p.block_m) + c * TC;
      const int lim = int(b * p.block_m) + p.block_m;
      f = -1;
      if (lane < TC && pos0 + lane < lim) f = __ldg(p.sorted_ids + pos0 + lane);
    };
    // the flat slot, or -1 for padding, a sentinel or an expert outside [0, E)
    auto valid_slot = [&](int e, int f) -> int {
      return (f >= 0 && f < p.n_slots && unsigned(e) < unsigned(p.E)) ? f : -1;
    };
    struct Group {
      int64_t v;              // worker index
      int64_t u, uend;        // its remaining units [u, uend)
      int e, nt;              // the current piece's item
      int ks, ksend;          // next stage of the current piece, and its end
      bool in_piece, done;
      uint32_t nitem;         // descriptors published to the group
      int64_t nw;             // the item whose metadata is prefetched below (-1: none)
      int ne, npos, nf;
    };
    // the group's next piece: item w, stages [ks0, ks0 + len); false when none is left
    auto peek = [&](const Group& G, int64_t& w, int& ks0, int& len) -> bool {
      if (G.u >= G.uend) return false;
      w = div_fast(G.u, KS);
      ks0 = int(G.u - w * KS);
      len = int(min(int64_t(KS - ks0), G.uend - G.u));
      return true;
    };
    // metadata of the group's next piece, loaded now so that its latency hides under
    // the streaming of the current one
    auto prefetch = [&](Group& G) {
      int64_t w;
      int ks0, len;
      G.nw = -1;
      if (peek(G, w, ks0, len)) {
        G.nw = w;
        load_meta(w, G.ne, G.npos, G.nf);
      }
    };
    auto init_group = [&](Group& G, int g) {
      // the CTA's two groups are workers blockIdx.x and blockIdx.x + gridDim.x: far apart in
      // the weights (neighbouring workers, which hand partial sums over, sit in different CTAs)
      G.v = int64_t(g) * gridDim.x + blockIdx.x;
      G.u = G.v < PS ? range_start(G.v) : RU;
      G.uend = G.v < PS ? range_start(G.v + 1) : RU;
      G.in_piece = false;
      G.done = false;
      G.nitem = 0;
      G.e = G.nt = G.ks = G.ksend = 0;
      G.ne = G.npos = G.nf = 0;
      prefetch(G);
    };
    // publishes one descriptor to group g's ring
    auto publish = [&](Group& G, int g, int e, int nt, int pos0, int fval, int ks0, int nks, int kind,
                       int64_t vlast, bool end) -> bool {
      const uint32_t ds = g * kDescRingG + G.nitem % kDescRingG;
      if (G.nitem >= kDescRingG &&
          !mbar_wait(&dempty[ds], ((G.nitem / kDescRingG) - 1) & 1, abort_v, p.status))
        return false;
      ItemDesc* d = &descs[ds];
      if (lane < TC) d->f[lane] = fval;
      if (lane == 0) {
        d->e = e; d->nt = nt; d->pos0 = pos0; d->end = end ? 1 : 0;
        d->ks0 = ks0; d->nks = nks; d->kind = kind; d->v = int(G.v); d->vlast = int(vlast);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dfull[ds]);
      ++G.nitem;
      return true;
    };
    // takes the group's next piece with routed rows and publishes it; false when none is
    // left (done) or on abort (ok = false)
    auto next_piece = [&](Group& G, int g, bool& ok) -> bool {
      int64_t w;
      int ks0, len;
      while (peek(G, w, ks0, len)) {
        G.u += len;
        int e, pos0, fval;
        if (w == G.nw) {
          e = G.ne;
          pos0 = G.npos;
          fval = G.nf;
        } else {
          load_meta(w, e, pos0, fval);
        }
        prefetch(G);
        fval = valid_slot(e, fval);
        if (__ballot_sync(0xffffffffu, fval >= 0) == 0) continue;  // nothing routed here
        const bool head = ks0 == 0, tail = ks0 + len == KS;
        const int kind = head ? (tail ? kPieceFull : kPieceOwner) : kPiecePart;
        const int64_t vlast = kind == kPieceOwner ? worker_of((w + 1) * KS - 1) : G.v;
        const int nt = int(w - div_fast(w, NTILES) * NTILES);
        if (!publish(G, g, e, nt, pos0, fval, ks0, len, kind, vlast, false)) {
          ok = false;
          return false;
        }
        G.e = e;
        G.nt = nt;
        G.ks = ks0;
        G.ksend = ks0 + len;
        G.in_piece = true;
        return true;
      }
      G.done = true;
      return false;
    };
    // streams stage ks of the item on expert e, tile nt: one bulk copy of up to KTS tiles
    auto stream_stage = [&](int e, int nt, int ks) -> bool {
      const uint32_t slot = stage % NSTAGE;
      if (stage >= uint32_t(NSTAGE) &&
          !mbar_wait(&empty[slot], ((stage / NSTAGE) - 1) & 1, abort_v, p.status))
        return false;
      const int kt0 = ks * KTS;
      const int ntl = min(KTS, KT - kt0);
      if (lane == 0) {
        uint8_t* st = stages + slot * kStageBytes;
        const uint64_t tile0 = (uint64_t(e) * NTILES + uint64_t(nt)) * KT;
        mbar_arrive_expect_tx(&full[slot], uint32_t(ntl) * kTileBytes);
        bulk_g2s_hint(st, p.tiles + (tile0 + kt0) * kTileBytes, uint32_t(ntl) * kTileBytes, &full[slot], pol_w);
      }
      ++stage;
      return true;
    };
    // a stage slot of a group whose range is exhausted while the other group still streams:
    // no copy and no consumer (the producer frees it itself), so that stage s keeps
    // belonging to group s % 2
    auto dummy_stage = [&]() -> bool {
      const uint32_t slot = stage % NSTAGE;
      if (stage >= uint32_t(NSTAGE) &&
          !mbar_wait(&empty[slot], ((stage / NSTAGE) - 1) & 1, abort_v, p.status))
        return false;
      if (lane == 0) {
        mbar_arrive(&full[slot]);
        mbar_arrive_cnt(&empty[slot], 8);
      }
      __syncwarp();
      ++stage;
      return true;
    };
    // the stage of group G (then the other group O has the next one)
    auto step = [&](Group& G, int g, Group& O, bool& ok) {
      if (!G.in_piece && !G.done) next_piece(G, g, ok);
      if (!ok) return;
      if (G.in_piece) {
        ok = stream_stage(G.e, G.nt, G.ks);
        if (++G.ks == G.ksend) G.in_piece = false;
      } else if (!O.done || O.in_piece) {
        ok = dummy_stage();
      }
    };
    Group g0, g1;
    init_group(g0, 0);
    init_group(g1, 1);
    bool ok = true;  // false once a wait gave up (abort)
    while (ok) {
      step(g0, 0, g1, ok);
      if (!ok || (g0.done && !g0.in_piece && g1.done && !g1.in_piece)) break;
      step(g1, 1, g0, ok);
      if (g0.done && !g0.in_piece && g1.done && !g1.in_piece) break;
    }
    // every stage is issued: the next kernel may launch and take SMs as CTAs here finish
    grid_dep_trigger();
    // an end marker for each group
    bool ok0 = true, ok1 = true;
    if (ok) ok0 = publish(g0, 0, 0, 0, 0, -1, 0, 0, kPieceFull, 0, true);
    if (ok) ok1 = publish(g1, 1, 0, 0, 0, -1, 0, 0, kPieceFull, 0, true);
    (void)ok0;
    (void)ok1;
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
  const int grp = cw >> 3;             // consumer group = worker grp * gridDim.x + blockIdx.x
  const int rb = cw & 7;               // 16-row block inside the tile
  const int g = lane >> 2, t = lane & 3;
  uint32_t k = 0;                      // this group's stages so far: its k-th is stage 2k + grp
  for (uint32_t it = 0;; ++it) {
    const uint32_t ds = grp * kDescRingG + it % kDescRingG;
    if (!mbar_wait(&dfull[ds], (it / kDescRingG) & 1, abort_v, p.status)) return;
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

    // the accumulator chains summed
    auto reduce = [&](float (&accs)[NT8][4]) {
#pragma unroll
      for (int i = 0; i < NT8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v = 0.f;
#pragma unroll
          for (int q = 0; q < NSET; ++q) v += acc[i][q][c];
          accs[i][c] = v;
        }
    };
    // ---- epilogue of the item's 128-row tile `ntile`
    auto epilogue = [&](const float (&accs)[NT8][4], int ntile) {
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

    for (int q = 0; q < d.nks; ++q, ++k) {
      const int ks = d.ks0 + q;
      const uint32_t s = 2 * k + uint32_t(grp);
      const uint32_t slot = s % NSTAGE;
      if (!mbar_wait(&full[slot], (s / NSTAGE) & 1, abort_v, p.status)) return;
      const int ntl = min(KTS, KT - ks * KTS);
      // plain shared loads (ordered after the wait by its memory clobber) so the compiler
      // can schedule them ahead of the dequantisation and the MMAs
      const uint8_t* stg = stages + slot * kStageBytes;
      // software-pipelined over the stage's tiles: tile i + 1's codes are loaded from shared
      // memory before tile i is dequantised, so their latency overlaps the math
      TileCodes cur = load_tile_codes(stg, 0, rb, lane);
      for (int i = 0; i < ntl; ++i) {
        TileCodes nxt = cur;
        if (i + 1 < ntl) nxt = load_tile_codes(stg, i + 1, rb, lane);
        uint4 xv[4][NT8];
        load_tile_x<NT8>(xv, xrow, (ks * KTS + i) * kTileK);
        consume_tile<NT8, NSET>(cur, xv, acc, (i & 1) * 2);
        cur = nxt;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    float accs[NT8][4];
    reduce(accs);
    if (d.kind == kPiecePart) {
      // a later part of an item: leave the FP32 partial for the worker that finishes it
      float* dst = p.partial + ((int64_t(d.v) * 8 + rb) * 32 + lane) * (NT8 * 4);
#pragma unroll
      for (int n8 = 0; n8 < NT8; ++n8)
        __stcg(reinterpret_cast<float4*>(dst + n8 * 4), make_float4(accs[n8][0], accs[n8][1], accs[n8][2], accs[n8][3]));
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release_gpu(p.flags + int64_t(d.v) * 8 + rb, 1u);
    } else {
      if (d.kind == kPieceOwner) {
        // the item's first part, reached last in this worker's range: add the partials of
        // the workers holding its other stages, in worker order (deterministic)
        for (int v2 = d.v + 1; v2 <= d.vlast; ++v2) {
          uint32_t* fl = p.flags + int64_t(v2) * 8 + rb;
          if (lane == 0 && ld_acquire_gpu(fl) == 0u) {
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_gpu(fl) == 0u) {
              if (*abort_v) break;
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_v = 1;
                atomicOr(p.status, CHORD_DEV_TIMEOUT);
                break;
              }
              __nanosleep(200);
            }
          }
          __syncwarp();
          if (*abort_v) return;
          const float* src = p.partial + ((int64_t(v2) * 8 + rb) * 32 + lane) * (NT8 * 4);
#pragma unroll
          for (int n8 = 0; n8 < NT8; ++n8) {
            const float4 pv = __ldcg(reinterpret_cast<const float4*>(src + n8 * 4));
            accs[n8][0] += pv.x;
            accs[n8][1] += pv.y;
            accs[n8][2] += pv.z;
            accs[n8][3] += pv.w;
          }
          __syncwarp();
          if (lane == 0) *fl = 0u;  // ready for the next launch
        }
      }
      epilogue(accs, d.nt);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&dempty[ds]);
  }
}

template <int EPI, int TC>
cudaError_t launch_one(const StreamParams& p, int grid, bool pdl, cudaStream_t stream) {
  auto kern = stream_gemm_kernel<EPI, TC>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<TC>::kBytes);
  if (err != cudaSuccess) return err;
  err = launch_pdl(pdl, kern, dim3(grid), dim3(kThreads), size_t(Smem<TC>::kBytes), stream, p);
  count_launches(1);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// K of at least one stage: this file's stream-K kernel; shorter K: the round-robin kernel
template <int EPI>
cudaError_t launch_tc(const StreamParams& p, int tc, int num_sms, bool pdl, cudaStream_t stream) {
  if (p.K < kShortK) return launch_stream_gemm_short(EPI, p, tc, num_sms, pdl, stream);
  const int grid = min(num_sms, kMaxStreamCtas);
  switch (tc) {
    case 8: return launch_one<EPI, 8>(p, grid, pdl, stream);
    case 16: return launch_one<EPI, 16>(p, grid, pdl, stream);
    default: return launch_one<EPI, 32>(p, grid, pdl, stream);
  }
}

}  // namespace
}  // namespace stream

using namespace stream;

cudaError_t launch_stream_gemms(const ForwardArgs& a, cudaStream_t stream, cudaEvent_t first, cudaEvent_t mid) {
  const int tc = stream_token_chunk(a.block_m);
  StreamParams p{};
  p.ntp = a.ntp;
  p.sorted_ids = a.sorted_ids;
  p.expert_ids = a.expert_ids;
  p.block_m = a.block_m;
  p.n_slots = a.T * a.topk;
  p.topk = a.topk;
  p.cap = a.cap;
  p.a_out = a.a;
  p.y_out = a.y;
  p.topk_weights = a.topk_weights;
  p.I = a.I;
  p.H = a.H;
  p.E = a.E;
  p.status = a.status;

  // gate_up: W13 [E, 2I, H], activations x [T, H]
  p.blob = a.w13;
  p.tiles = a.w13 + blob_tiles_offset();
  p.N = 2 * a.I;
  p.K = a.H;
  p.role = CHORD_ROLE_GATE_UP;
  p.act = a.x;
  p.act_ld = a.H;
  p.flags = a.stream_flags;
  p.partial = a.stream_partial;
  cudaError_t err = first ? record_timing_event(first, stream) : cudaSuccess;
  if (err != cudaSuccess) return err;
  err = launch_tc<kGateUp>(p, tc, a.num_sms, a.pdl, stream);
  if (err != cudaSuccess) return err;
  if (mid && (err = record_timing_event(mid, stream)) != cudaSuccess) return err;

  // down: W2 [E, H, I], activations a [cap, I]
  p.blob = a.w2;
  p.tiles = a.w2 + blob_tiles_offset();
  p.N = a.H;
  p.K = a.I;
  p.role = CHORD_ROLE_DOWN;
  p.act = a.a;
  p.act_ld = a.I;
  p.flags = a.stream_flags + kMaxStreamWorkers * 8;
  p.partial = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.stream_partial) + a.stream_partial_bytes);
  return launch_tc<kDown>(p, tc, a.num_sms, a.pdl, stream);
}

cudaError_t launch_stream_grouped(const GroupedArgs& g, cudaStream_t stream) {
  // one token chunk per routing unit
  if (g.bm != 8 && g.bm != 16 && g.bm != 32) return cudaErrorInvalidValue;
  const int tc = g.bm;
  StreamParams p{};
  p.ntp = g.ntp;
  p.sorted_ids = g.sorted_ids;
  p.expert_ids = g.expert_ids;
  p.block_m = g.bm;
  p.n_slots = g.rows;  // sorted_ids holds x rows
  p.topk = 1;
  p.cap = g.cap;
  p.out = g.out;
  p.E = g.E;
  p.status = g.status;
  p.blob = g.w;
  p.tiles = g.w + blob_tiles_offset();
  p.N = g.N;
  p.K = g.K;
  p.role = g.role;
  p.act = g.x;
  p.act_ld = g.K;
  p.flags = g.stream_flags;
  p.partial = g.stream_partial;
  return launch_tc<kPlain>(p, tc, g.num_sms, false, stream);
}

}  // namespace chord
