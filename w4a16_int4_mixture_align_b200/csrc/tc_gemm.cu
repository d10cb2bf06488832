// tc_gemm.cu -- tensor-core (tcgen05) W4A16 grouped GEMMs for many tokens per expert.
//
// Above a few dozen routed tokens per expert the layer is bound by the tensor cores, and
// the int4 dequantisation must be paid once per weight tile and shared by as many tokens
// as possible. The Chord blog's H200 prefill kernels overlap the dequantisation of the
// next K slice with the in-flight WGMMA group ("H200 Prefill und TP8": batched wait<1>
// pipelining) and size block_m from the tokens routed per expert. On sm_100a the MMA is
// asynchronous by construction, so the overlap becomes warp specialisation, and the
// kernel runs on CTA pairs (clusters of two, tcgen05 cta_group::2):
//
//   An item is (routing block b of up to 256 rows, a 256-row weight tile). CTA rank r of
//   the pair owns the weight rows of 128-row tile 2*nt2 + r and, of the block's N routed
//   rows (rounded up to 16), rows [r*N/2, (r+1)*N/2) of the activation operand. One
//   M = 256 MMA then multiplies each CTA's 128 weight rows with all N rows, so each SM
//   fetches only half of the activation bytes a single-CTA M = 128 tile would (those
//   bytes, about 32 per MMA cycle per SM, come from L2 and their latency is what the
//   rings must cover).
//
//   warp 0      activation producer (both CTAs): per 128-wide K step one TMA request
//               for this CTA's half of the block's rows, two 64-column chunks of them
//               (a 3-D box over the row-major activations viewed as {64 columns, rows,
//               chunks}, 128-byte swizzle, landing chunk-major), into its B ring; the copies of both CTAs complete on the B
//               barrier of rank 0. One request per step matters: each TMA issue holds the
//               issuing thread for a few hundred cycles, so the box height equals the
//               half-block (a tensor map per height, 8..128 rows). The rows are contiguous
//               because the activations are in routing order: the intermediate of the down
//               projection is written that way, and the gate_up input is permuted first.
//   warp 2      weight producer (both CTAs): one bulk copy of the packed codes + scales of
//               two 128-wide K tiles of this CTA's weight tile per raw stage.
//   warps 3..18 dequant (both CTAs): raw int4 -> bf16 (subtract 8, then scale) into the
//               A ring in the UMMA K-major 128-byte-swizzle layout, one row per lane, one
//               128-wide K tile per A stage (the A and B rings step together); arrivals
//               go to rank 0's A barrier. Sixteen warps, because the MMA waits on the
//               latency of this dependent int -> bf16 chain rather than on issue slots.
//   warp 1      MMA (rank 0, one thread): tcgen05.mma.cta_group::2 (M = 256, N = the
//               block's routed rows rounded up to 16, K = 16) into one of two TMEM
//               accumulators of 256 columns; tcgen05.commit multicast to both CTAs frees
//               the ring stages and publishes the accumulator.
//   warps 19..26 epilogue (both CTAs, two per TMEM lane quadrant, alternate 16-column
//               chunks): tcgen05.ld of this CTA's 128 accumulator rows; SiLU(gate)*up
//               written to the bf16 intermediate (gate_up), or the fp32 expert
//               output written by sorted position in 128-column blocks (down; the combine
//               applies the top-k weight).
//               Double buffering lets it overlap the next item.
//
// The A and B rings step together (one 128-K step per stage), so they share one barrier
// ring indexed by step (depth D = the deeper of the two): step_full[j % D] collects the
// 32 dequant-warp arrivals of both CTAs and the activation bytes of step j, and one
// multicast commit per step frees step_empty[j % D] for both rings. Neither producer can
// fill step j + D before step j is done (D is at least either ring's depth), so a phase
// never receives arrivals from two steps. One wait and one commit per step keep the MMA
// thread's own work short: its MMA issue blocks for about the tensor time, so whatever
// else it does between steps is a bubble in the tensor pipe.
//
// When the weight matrix has an odd number of 128-row tiles, rank 1 of the last pair
// tile computes on stale shared memory and writes nothing.
//
// Operand orientation follows the blog's decode profile (dequantised weights in the
// MMA-M slot, tokens in N): one dequantised weight tile serves every token of a block.
// All waits are bounded; on timeout the CTA raises CHORD_DEV_TIMEOUT and unwinds after
// waiting (bounded) for its copies and MMAs in flight, then frees TMEM. Both CTAs of a
// pair meet at a cluster barrier before TMEM is freed and before either exits, so no
// remote arrival or copy can target a CTA that has left.
#include <cuda.h>

#include <mutex>

#include "tc_common.cuh"

namespace chord {
namespace {

constexpr int kRawTiles = 2;      // 128-wide K tiles per raw stage (one bulk copy)
constexpr int kMaxRawStages = 8;  // upper bound of the raw weight ring (runtime sized, >= 3)
constexpr int kMaxStages = 8;     // upper bound of the A and B rings (runtime sized)
constexpr int kMaxN = 256;
constexpr int kDescRingTC = 8;
constexpr int kDequantWarps = 16;
constexpr int kEpiWarps = 8;
constexpr int kTcThreads = 32 * (3 + kDequantWarps + kEpiWarps);
constexpr int kFirstDequantWarp = 3;
constexpr int kFirstEpiWarp = kFirstDequantWarp + kDequantWarps;
constexpr int kBChunks = 2;        // 64-column chunks per activation request (one 128-K step)
constexpr int kNumBoxMaps = 16;    // activation box heights 8, 16, ..., 128 rows

constexpr int kAStageBytes = 128 * 128 * 2;   // 128 rows x one 128-K tile (two SW128 halves)
constexpr int kAHalfBytes = kAStageBytes / 2;
constexpr int kRawStageBytes = kRawTiles * kTileBytes;
constexpr int kBInFlightBytes = 96 * 1024;  // activation bytes to keep in flight per CTA

struct TcDesc {
  int e, nt, pos0, nvalid, end, phantom, pad[2];
};
// fixed part (from the 1024-aligned base): descriptors, barriers, TMEM slot; then rings
constexpr int kOffDesc = 0;
constexpr int kOffBar = kOffDesc + kDescRingTC * int(sizeof(TcDesc));
constexpr int kNumBars = 2 * kMaxRawStages + 4 * kMaxStages + 4 + 2 * kDescRingTC;
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kOffRings = 1024;
static_assert(kOffTmemSlot + 16 <= kOffRings, "fixed part");
constexpr int kSmemLimit = 232448 - 1024;  // 227 KiB opt-in per CTA, minus static shared

// Ring geometry for a launch whose largest MMA N is nmax (each CTA holds nmax/2 rows x
// kBChunks chunks of a B stage). A and B stages both cover one 128-wide K step.
struct TcRings {
  int a_stages, b_stages, raw_stages, b_stage_bytes, off_a, off_b, off_raw, smem_bytes;
};
__host__ __device__ inline TcRings tc_rings(int nmax) {
  auto clamp = [](int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); };
  TcRings r;
  r.b_stage_bytes = (nmax / 2) * 128 * kBChunks;
  const int avail = kSmemLimit - 1024 - kOffRings;
  // enough activation stages to cover the L2 latency and a two-deep A ring; then as many
  // raw weight stages as fit (the weight copies wait on HBM, so with small activation
  // tiles the spare room goes to weights in flight); then what is left to A, then B gets
  // what remains (fewer stages than the latency target when the tiles are large)
  int bs = clamp((kBInFlightBytes + r.b_stage_bytes - 1) / r.b_stage_bytes, 2, kMaxStages);
  const int rs = clamp((avail - bs * r.b_stage_bytes - 2 * kAStageBytes) / kRawStageBytes, 3, kMaxRawStages);
  const int as = clamp((avail - bs * r.b_stage_bytes - rs * kRawStageBytes) / kAStageBytes, 2, kMaxStages);
  bs = clamp((avail - as * kAStageBytes - rs * kRawStageBytes) / r.b_stage_bytes, 2, kMaxStages);
  r.a_stages = as;
  r.b_stages = bs;
  r.raw_stages = rs;
  r.off_a = kOffRings;
  r.off_b = r.off_a + as * kAStageBytes;
  r.off_raw = r.off_b + bs * r.b_stage_bytes;
  r.smem_bytes = r.off_raw + rs * kRawStageBytes + 1024;  // + base alignment slack
  return r;
}

// kGateUp: SiLU(gate) * up into a; kDown: fp32 y by position; kPlain: bf16 out[row, n]
// (grouped operators).
enum Epi { kGateUp = 0, kDown = 1, kPlain = 2 };

// Position in a ring of runtime size: slot index and the phase parity of its barriers.
struct RingPos {
  uint32_t slot = 0, phase = 0, count = 0;
  __device__ __forceinline__ void next(uint32_t stages) {
    ++count;
    if (++slot == stages) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

struct TcParams {
  const uint8_t* tiles;
  const uint8_t* blob;
  int N, K, E, role;
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntp;
  int block_m;
  int64_t n_slots;
  int topk;
  int64_t cap;
  const int32_t* block_row0;  // activation row of each block's first position (grouped), or null
  uint16_t* out;              // kPlain output [rows, N]
  uint16_t* a_out;
  float* y_out;
  const float* topk_weights;
  int I, H;
  uint32_t* status;
  TcRings rings;
};

// Dequantises half hk (64 K) of one row's 128-K tile into one SW128 half of an A stage
// (UMMA K-major, 128-byte swizzle). Lane (g, t) owns row r: `c` holds its four code
// words (K slices j = 0..3 at offset 8t), `sp` the two scales of slices 2hk, 2hk+1. The
// slice order alternates with g so the eight lanes of each 16-byte store phase hit eight
// distinct bank groups.
template <int HK>
__device__ __forceinline__ void dequant_row_half(const uint4& c, uint32_t sp, uint32_t a_stage, int r,
                                                 int g, int t) {
  const uint32_t w0 = HK ? c.z : c.x;
  const uint32_t w1 = HK ? c.w : c.y;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int jj = (q + g) & 1;
    uint32_t o[4];
    dequant8(jj ? w1 : w0, bf16_splat_half(sp, jj), o);
    const int ch = 4 * jj + t;
    sts128(a_stage + (r >> 3) * 1024 + (r & 7) * 128 + ((ch ^ (r & 7)) << 4), o);
  }
}

// Tensor maps of the K-blocked activation tensor [K/64][cap][64], one per box height
// 8 * (i + 1) rows, box {64 columns, height, kBChunks chunks}.
struct BoxMaps {
  CUtensorMap m[kNumBoxMaps];
};

template <int EPI>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ BoxMaps maps, TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled operand stages (the same offset in both CTAs)
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  const int AS = p.rings.a_stages, BS = p.rings.b_stages;
  const uint32_t RS = uint32_t(p.rings.raw_stages);
  const int DS = AS > BS ? AS : BS;  // depth of the step barrier ring
  const int b_stage_bytes = p.rings.b_stage_bytes;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + kMaxRawStages;
  uint64_t* step_full = raw_empty + kMaxRawStages;  // [D] used in rank 0: dequant arrivals + copies
  uint64_t* step_empty = step_full + kMaxStages; // [D] one multicast commit per step
  uint64_t* spare = step_empty + kMaxStages;     // [2 * kMaxStages] unused
  uint64_t* acc_full = spare + 2 * kMaxStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;            // [2], used in rank 0: both epilogues
  uint64_t* dfull = acc_empty + 2;               // [kDescRingTC]
  uint64_t* dempty = dfull + kDescRingTC;        // [kDescRingTC]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmemSlot);
  TcDesc* descs = reinterpret_cast<TcDesc*>(smem + kOffDesc);
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
    for (int s = 0; s < p.rings.raw_stages; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kDequantWarps);
    }
    // descriptor consumers: dequant, epilogue, weight producer and (rank 0) the MMA thread
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&step_full[s], 2 * kDequantWarps + 1);  // dequant warps of both CTAs + rank 0's copy
      mbar_init(&step_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    for (int d = 0; d < kDescRingTC; ++d) {
      mbar_init(&dfull[d], 1);
      mbar_init(&dempty[d], kDequantWarps + kEpiWarps + 1 + (leader ? 1 : 0));
    }
    fence_barrier_init();
  }
  __syncthreads();
  // both CTAs of a pair read the same header, so they leave here together or not at all
  if (abort_flag) return;
  cluster_sync_all();  // the peer's barriers are initialised before anything arrives on them
  if (warp == 1) tmem_alloc_pair(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = &abort_flag;

  const int KT = p.K / kTileK;        // 128-wide raw steps
  const int NTILES = p.N / kTileN;
  const int NT2 = (NTILES + 1) / 2;   // 256-row pair tiles
  const int64_t cid = cluster_id_x(), ncl = num_clusters_x();

  if (warp == 0) {
    // ----------------------------------------------------------------- activation producer
    const int ntp = routed_positions(p.ntp, p.block_m, p.cap, p.status);
    const int64_t nblocks = ntp / p.block_m;
    const int64_t items = nblocks * NT2;
    const uint64_t pol_a = policy_evict_last();
    const uint32_t step_full_l = cluster_addr(step_full, 0);
    uint32_t nitem = 0;
    RingPos bpos, fill, lag;  // B data slot; step barrier of the fill; step the slot last held
    bool ok = true;
    // routing metadata of item w (its expert and the flat slots of this lane's 8 rows),
    // loaded one item ahead so the latency overlaps the current item's streaming
    auto load_meta = [&](int64_t w, int& e, int& r0, int (&f)[kMaxN / 32]) {
      e = -1;
      r0 = 0;
#pragma unroll
      for (int i = 0; i < kMaxN / 32; ++i) f[i] = -1;
      if (w >= items) return;
      const int64_t b = w / NT2;
      e = __ldg(p.expert_ids + b);
      r0 = p.block_row0 ? __ldg(p.block_row0 + b) : int(b * p.block_m);
      const int pos0 = int(b * p.block_m);
#pragma unroll
      for (int i = 0; i < kMaxN / 32; ++i) {
        const int r = lane + 32 * i;
        if (r < p.block_m) f[i] = __ldg(p.sorted_ids + pos0 + r);
      }
    };
    int e_next, r0_next, f_next[kMaxN / 32];
    load_meta(cid, e_next, r0_next, f_next);
    for (int64_t w = cid; ok; w += ncl) {
      const bool end = w >= items;
      int e = e_next, nt = 0, pos0 = 0, nvalid = 0;
      const int r0 = r0_next;
      int fcur[kMaxN / 32];
#pragma unroll
      for (int i = 0; i < kMaxN / 32; ++i) fcur[i] = f_next[i];
      load_meta(w + ncl, e_next, r0_next, f_next);
      if (!end) {
        nt = int(w % NT2) * 2 + int(rank);
        pos0 = int((w / NT2) * p.block_m);
        if (unsigned(e) < unsigned(p.E)) {
#pragma unroll
          for (int i = 0; i < kMaxN / 32; ++i)
            if (fcur[i] >= 0 && fcur[i] < p.n_slots) nvalid = lane + 32 * i + 1;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) nvalid = max(nvalid, __shfl_xor_sync(0xffffffffu, nvalid, o));
        if (nvalid == 0) continue;  // both CTAs see the same rows and skip together
      }
      const uint32_t ds = nitem % kDescRingTC;
      if (nitem >= kDescRingTC &&
          !mbar_wait(&dempty[ds], ((nitem / kDescRingTC) - 1) & 1, abort_v, p.status))
        break;
      if (lane == 0) {
        descs[ds].e = e;
        descs[ds].nt = nt;
        descs[ds].pos0 = pos0;
        descs[ds].nvalid = nvalid;
        descs[ds].end = end ? 1 : 0;
        descs[ds].phantom = nt >= NTILES ? 1 : 0;
        mbar_arrive(&dfull[ds]);
      }
      ++nitem;
      if (end) break;
      __syncwarp();
      const int nmma = (nvalid + 15) & ~15;
      const int half = nmma >> 1;                 // rows per CTA, a multiple of 8
      const CUtensorMap* map = &maps.m[(half >> 3) - 1];
      const int row0 = r0 + int(rank) * half;
      for (int kb = 0; kb < KT; ++kb) {
        const uint32_t s = bpos.slot;
        // the slot's previous fill (BS steps ago) must have been consumed
        if (bpos.count >= uint32_t(BS)) {
          if (!mbar_wait(&step_empty[lag.slot], lag.phase, abort_v, p.status)) {
            ok = false;
            break;
          }
          lag.next(DS);
        }
        if (lane == 0) {
          // rank 0 expects the bytes of both halves; each CTA copies its own half
          if (leader) mbar_arrive_expect_tx(&step_full[fill.slot], uint32_t(nmma) * 128u * kBChunks);
          tma_box3d_pair(sbase + p.rings.off_b + s * b_stage_bytes, map, row0, kb * kBChunks,
                         step_full_l + fill.slot * 8u, pol_a);
        }
        bpos.next(BS);
        fill.next(DS);
      }
      __syncwarp();
    }
    // drain: rank 0 waits (bounded, ignoring abort) for the steps of the last min(BS,
    // fills) fills (both halves complete on its barriers), walking back from the current one
    if (lane == 0 && leader) {
      int dummy = 0;
      RingPos back = fill;
      const uint32_t n_back = fill.count < uint32_t(BS) ? fill.count : uint32_t(BS);
      for (uint32_t i = 0; i < n_back; ++i) {
        if (back.slot == 0) {
          back.slot = DS - 1;
          back.phase ^= 1u;
        } else {
          --back.slot;
        }
        mbar_wait(&step_full[back.slot], back.phase, &dummy, p.status);
      }
    }
  } else if (warp == 2) {
    // ----------------------------------------------------------------- weight producer
    const uint64_t pol_w = policy_evict_first();
    uint32_t rstage = 0;
    for (uint32_t it = 0;; ++it) {
      const uint32_t ds = it % kDescRingTC;
      if (!mbar_wait(&dfull[ds], (it / kDescRingTC) & 1, abort_v, p.status)) break;
      const TcDesc d = descs[ds];
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[ds]);
      if (d.end) break;
      const uint64_t tile0 = (uint64_t(d.e) * NTILES + d.nt) * KT;
      bool ok = true;
      for (int kt0 = 0; kt0 < KT; kt0 += kRawTiles) {
        const int ntl = min(kRawTiles, KT - kt0);
        const uint32_t rs = rstage % RS;
        if (rstage >= RS && !mbar_wait(&raw_empty[rs], ((rstage / RS) - 1) & 1, abort_v, p.status)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          if (d.phantom) {
            mbar_arrive(&raw_full[rs]);
          } else {
            uint8_t* st = smem + p.rings.off_raw + rs * kRawStageBytes;
            mbar_arrive_expect_tx(&raw_full[rs], uint32_t(ntl) * kTileBytes);
            bulk_g2s_hint(st, p.tiles + (tile0 + kt0) * kTileBytes, uint32_t(ntl) * kTileBytes, &raw_full[rs],
                          pol_w);
          }
        }
        ++rstage;
      }
      __syncwarp();
      if (!ok) break;
    }
    // drain: wait (bounded, ignoring abort) for the copies still in flight
    if (lane == 0) {
      int dummy = 0;
      for (uint32_t s = (rstage > RS ? rstage - RS : 0); s < rstage; ++s)
        mbar_wait(&raw_full[s % RS], (s / RS) & 1, &dummy, p.status);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA issuer
    if (leader && lane == 0) {
      RingPos apos, bpos, step;
      uint64_t* last_bar = nullptr;
      uint32_t last_parity = 0;
      for (uint32_t it = 0;; ++it) {
        const uint32_t ds = it % kDescRingTC;
        if (!mbar_wait(&dfull[ds], (it / kDescRingTC) & 1, abort_v, p.status)) break;
        const TcDesc d = descs[ds];
        mbar_arrive(&dempty[ds]);
        if (d.end) break;
        const uint32_t buf = it & 1;
        if (it >= 2 && !mbar_wait(&acc_empty[buf], ((it >> 1) - 1) & 1, abort_v, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * 256;
        const int nmma = (d.nvalid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_m256(nmma);
        // descriptor increments: the start-address field holds address / 16
        const uint64_t b_chunk_inc = uint64_t(nmma >> 1) * 128u / 16u;  // one chunk of this CTA's rows
        const uint64_t a_half_inc = uint64_t(kAHalfBytes) / 16u;
        bool ok = true;
        for (int kb = 0; kb < KT; ++kb) {
          if (!mbar_wait(&step_full[step.slot], step.phase, abort_v, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(sbase + p.rings.off_a + apos.slot * kAStageBytes);
          const uint64_t bd = sw128_kmajor_desc(sbase + p.rings.off_b + bpos.slot * b_stage_bytes);
#pragma unroll
          for (int h = 0; h < kBChunks; ++h) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc2_mma(d_tmem, ad + h * a_half_inc + k * 2, bd + h * b_chunk_inc + k * 2, idesc,
                      (kb > 0 || h > 0 || k > 0) ? 1u : 0u);
          }
          tc2_commit_both(&step_empty[step.slot]);
          last_bar = &step_empty[step.slot];
          last_parity = step.phase;
          step.next(DS);
          apos.next(AS);
          bpos.next(BS);
        }
        if (!ok) break;
        tc2_commit_both(&acc_full[buf]);
      }
      // make sure no MMA is still writing TMEM before it is freed
      if (last_bar) {
        int dummy = 0;
        mbar_wait(last_bar, last_parity, &dummy, p.status);
      }
    }
  } else if (warp < kFirstEpiWarp) {
    // ----------------------------------------------------------------- dequant
    const int w = warp - kFirstDequantWarp;
    const int rb = w >> 1, hrow = w & 1;          // 16-row block, upper or lower 8 rows
    const int g = lane >> 2, t = lane & 3;
    const int row = rb * 16 + 8 * hrow + g;
    const uint32_t step_full_l = cluster_addr(step_full, 0);
    uint32_t rstage = 0;
    RingPos apos, fill, lag;  // A data slot; step barrier of the fill; step the slot last held
    for (uint32_t it = 0;; ++it) {
      const uint32_t ds = it % kDescRingTC;
      if (!mbar_wait(&dfull[ds], (it / kDescRingTC) & 1, abort_v, p.status)) break;
      const int end = descs[ds].end;
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[ds]);
      if (end) break;
      bool ok = true;
      for (int kt0 = 0; kt0 < KT && ok; kt0 += kRawTiles) {
        const int ntl = min(kRawTiles, KT - kt0);
        const uint32_t rs = rstage % RS;
        if (!mbar_wait(&raw_full[rs], (rstage / RS) & 1, abort_v, p.status)) { ok = false; break; }
        const uint32_t raw = sbase + p.rings.off_raw + rs * kRawStageBytes;
        for (int tl = 0; tl < ntl; ++tl) {
          // this lane's share of the tile: four code words and four group scales of its row
          const uint32_t tb = raw + tl * kTileBytes;
          const uint4 c = lds128(tb + rb * 1024 + hrow * 512 + g * 64 + code_slot(g, t) * 16);
          const uint2 sc = lds64(tb + kTileCodeBytes + rb * 128 + g * 16 + hrow * 8);
          const uint32_t s = apos.slot;
          // the slot's previous fill (AS steps ago) must have been consumed
          if (apos.count >= uint32_t(AS)) {
            if (!mbar_wait(&step_empty[lag.slot], lag.phase, abort_v, p.status)) {
              ok = false;
              break;
            }
            lag.next(DS);
          }
          const uint32_t a_stage = sbase + p.rings.off_a + s * kAStageBytes;
          dequant_row_half<0>(c, sc.x, a_stage, row, g, t);
          dequant_row_half<1>(c, sc.y, a_stage + kAHalfBytes, row, g, t);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(step_full_l + fill.slot * 8u);
          apos.next(AS);
          fill.next(DS);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[rs]);
        ++rstage;
      }
      if (!ok) break;
    }
  } else {
    // ----------------------------------------------------------------- epilogue
    const int q = warp & 3;                        // TMEM lane quadrant this warp may access
    const int half = (warp - kFirstEpiWarp) >> 2;  // which 16-column chunks (even / odd)
    const int r = q * 32 + lane;
    const uint32_t acc_empty_l = cluster_addr(acc_empty, 0);
    for (uint32_t it = 0;; ++it) {
      const uint32_t ds = it % kDescRingTC;
      if (!mbar_wait(&dfull[ds], (it / kDescRingTC) & 1, abort_v, p.status)) break;
      const TcDesc d = descs[ds];
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[ds]);
      if (d.end) break;
      const uint32_t buf = it & 1;
      // this item's flat slots, one per column, loaded before the accumulator wait so the
      // global-load latency hides under the mainloop
      int f_col[kMaxN / 32];
#pragma unroll
      for (int i = 0; i < kMaxN / 32; ++i) {
        const int c = lane + 32 * i;
        f_col[i] = -1;
        if (c < d.nvalid && !d.phantom) {
          const int f = __ldg(p.sorted_ids + d.pos0 + c);
          if (f >= 0 && f < p.n_slots) f_col[i] = f;
        }
      }
      if (!mbar_wait(&acc_full[buf], (it >> 1) & 1, abort_v, p.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + buf * 256;
      if (!d.phantom) {
#pragma unroll
        for (int cc = 0; cc < kMaxN / 16; ++cc) {
          const int c0 = cc * 16;
          if (c0 >= d.nvalid) break;
          if ((cc & 1) != half) continue;
          float v[16];
          tmem_ld16(taddr + c0, v);
          // column c0 + c lives in lane (c0 + c) % 32 of register set (c0 + c) / 32
          const int src_set = c0 >> 5;
          int f_set = f_col[0];
#pragma unroll
          for (int i = 1; i < kMaxN / 32; ++i)
            if (src_set == i) f_set = f_col[i];
          if (EPI == kGateUp) {
            const bool gate = (r & 15) < 8;
            const int i_col = d.nt * (kTileN / 2) + (r >> 4) * 8 + (r & 7);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float u = __shfl_down_sync(0xffffffffu, v[c], 8);
              const int f = __shfl_sync(0xffffffffu, f_set, (c0 & 31) + c);
              if (gate && f >= 0)
                p.a_out[int64_t(d.pos0 + c0 + c) * p.I + i_col] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(silu_mul(v[c], u)));
            }
          } else if (EPI == kPlain) {
            // out[row, n]: a warp stores 32 neighbouring columns (64 bytes) of one row
            const int n_col = d.nt * kTileN + r;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int f = __shfl_sync(0xffffffffu, f_set, (c0 & 31) + c);
              if (f >= 0)
                p.out[int64_t(f) * p.N + n_col] = __bfloat16_as_ushort(__float2bfloat16_rn(v[c]));
            }
          } else {
            // y by sorted position in 128-column blocks: this item's tile is one
            // contiguous run of 512-byte rows
            float* yb = p.y_out + (int64_t(d.nt) * p.cap + d.pos0 + c0) * kTileN + r;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int f = __shfl_sync(0xffffffffu, f_set, (c0 & 31) + c);
              if (f >= 0) yb[c * kTileN] = v[c];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_l + buf * 8u);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no MMA, copy or arrival of either CTA is still in flight
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ------------------------------------------------------------------------------------ host

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// Box maps of a row-major bf16 tensor [rows][K], viewed as 3-D {64 columns, rows,
// K/64 chunks} with strides {K*2, 128} bytes, so that a box {64, R, kBChunks} lands in
// shared memory chunk-major, [chunk][row][128 B]: the K-blocked tile the MMA reads. Map
// i has R = 8 * (i + 1) rows, 128-byte swizzle; rows past the end read as zero.
// Encoding sixteen maps costs host time, so the last few sets are kept, keyed by the
// tensor's address and shape (the workspace of a layer is reused call after call).
cudaError_t box_maps(BoxMaps* out, const void* base, int64_t rows, int K) {
  struct Entry {
    const void* base;
    int64_t rows;
    int K, dev;
    BoxMaps maps;
  };
  static std::mutex mu;
  static Entry cache[4];
  static int n_cache = 0, next_slot = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n_cache; ++i)
    if (cache[i].base == base && cache[i].rows == rows && cache[i].K == K && cache[i].dev == dev) {
      *out = cache[i].maps;
      return cudaSuccess;
    }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  BoxMaps maps;
  cuuint64_t dims[3] = {64, cuuint64_t(rows), cuuint64_t(K / 64)};
  cuuint64_t strides[2] = {cuuint64_t(K) * 2, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  for (int i = 0; i < kNumBoxMaps; ++i) {
    cuuint32_t box[3] = {64, cuuint32_t(8 * (i + 1)), cuuint32_t(kBChunks)};
    CUresult r = fn(&maps.m[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  Entry& e = cache[next_slot];
  e.base = base;
  e.rows = rows;
  e.K = K;
  e.dev = dev;
  e.maps = maps;
  next_slot = (next_slot + 1) % 4;
  if (n_cache < 4) ++n_cache;
  *out = maps;
  return cudaSuccess;
}

// Largest number of co-resident CTA pairs for this kernel and shared-memory size, per
// device (clusters must fit inside a GPC, so this can be below half the SM count).
template <int EPI>
int max_pairs(int smem_bytes, int max_ctas) {
  struct Entry {
    int dev, smem, pairs;
  };
  static std::mutex mu;
  static Entry cache[16];
  static int n_cache = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n_cache; ++i)
    if (cache[i].dev == dev && cache[i].smem == smem_bytes) return min(cache[i].pairs, max_ctas / 2);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(unsigned(max_ctas & ~1));
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = size_t(smem_bytes);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int pairs = 0;
  if (cudaOccupancyMaxActiveClusters(&pairs, tc_gemm_kernel<EPI>, &cfg) != cudaSuccess) return 0;
  if (n_cache < 16) cache[n_cache++] = Entry{dev, smem_bytes, pairs};
  return min(pairs, max_ctas / 2);
}

template <int EPI>
cudaError_t launch_one(const BoxMaps& maps, const TcParams& p, int max_ctas, cudaStream_t stream) {
  auto kern = tc_gemm_kernel<EPI>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  if (err != cudaSuccess) return err;
  const int pairs = max_pairs<EPI>(p.rings.smem_bytes, max_ctas);
  if (pairs < 1) return cudaErrorLaunchOutOfResources;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(unsigned(2 * pairs));
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = size_t(p.rings.smem_bytes);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, maps, p);
  count_launches(1);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemms(const ForwardArgs& a, cudaStream_t stream, cudaEvent_t first, cudaEvent_t mid) {
  TcParams p{};
  p.sorted_ids = a.sorted_ids;
  p.expert_ids = a.expert_ids;
  p.ntp = a.ntp;
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
  p.rings = tc_rings(min(kMaxN, (a.block_m + 15) & ~15));
  const int grid = a.num_sms;

  // gate_up: W13 [E, 2I, H]; B rows from the hidden states permuted into routing order
  cudaError_t err = launch_permute_rows(a, stream);
  if (err != cudaSuccess) return err;
  BoxMaps maps;
  err = box_maps(&maps, a.xs, a.cap, a.H);
  if (err != cudaSuccess) return err;
  p.blob = a.w13;
  p.tiles = a.w13 + blob_tiles_offset();
  p.N = 2 * a.I;
  p.K = a.H;
  p.role = CHORD_ROLE_GATE_UP;
  if (first && (err = record_timing_event(first, stream)) != cudaSuccess) return err;
  if ((err = launch_one<kGateUp>(maps, p, grid, stream)) != cudaSuccess) return err;
  if (mid && (err = record_timing_event(mid, stream)) != cudaSuccess) return err;

  // down: W2 [E, H, I]; B rows of the K-blocked intermediate a, already in routing order
  if ((err = box_maps(&maps, a.a, a.cap, a.I)) != cudaSuccess) return err;
  p.blob = a.w2;
  p.tiles = a.w2 + blob_tiles_offset();
  p.N = a.H;
  p.K = a.I;
  p.role = CHORD_ROLE_DOWN;
  return launch_one<kDown>(maps, p, grid, stream);
}

cudaError_t launch_tc_grouped(const GroupedArgs& g, cudaStream_t stream) {
  TcParams p{};
  p.sorted_ids = g.sorted_ids;
  p.expert_ids = g.expert_ids;
  p.block_row0 = g.block_row0;
  p.ntp = g.ntp;
  p.block_m = g.bm;
  p.n_slots = g.rows;  // sorted_ids holds x rows
  p.topk = 1;
  p.cap = g.cap;
  p.out = g.out;
  p.E = g.E;
  p.status = g.status;
  p.rings = tc_rings(min(kMaxN, g.bm));
  p.blob = g.w;
  p.tiles = g.w + blob_tiles_offset();
  p.N = g.N;
  p.K = g.K;
  p.role = g.role;
  BoxMaps maps;
  cudaError_t err = box_maps(&maps, g.x, g.rows, g.K);
  if (err != cudaSuccess) return err;
  return launch_one<kPlain>(maps, p, g.num_sms, stream);
}

}  // namespace chord
