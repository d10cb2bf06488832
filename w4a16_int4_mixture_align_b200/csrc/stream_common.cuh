// stream_common.cuh -- parameters and tile helpers shared by the two weight-streaming
// W4A16 GEMM kernels: stream_gemm.cu (stream-K work division, for K of at least one stage)
// and stream_gemm_short.cu (whole items in round-robin pairs, for K shorter than a stage).
//
// Both stream the repacked weight tiles through a shared-memory ring with bulk copies and
// dequantise them straight into the A fragments of mma.m16n8k16 (weights in the MMA-M
// slot, routed tokens as N: the Chord blog's decode profile, "H200 und Blackwell
// indexierter Decode").
#pragma once

#include "chord_internal.cuh"

namespace chord {
namespace stream {

constexpr int kConsumerWarps = 16;          // two groups of 8
constexpr int kThreads = 32 * (1 + kConsumerWarps);
constexpr int kMaxTC = 32;                  // token columns of an item: 8, 16 or 32
constexpr int kKTS = 4;                     // 128-wide K tiles per stage (one bulk copy)
constexpr int kStageBytes = kKTS * kTileBytes;
constexpr int kMaxDynSmem = 232448 - 1024;  // 227 KiB opt-in per CTA, minus the static shared memory
// K below one stage: an item is a single stage covering several row tiles
constexpr int kShortK = kKTS * kTileK;

// kGateUp: SiLU(gate) * up into a; kDown: fp32 y by flat slot; kPlain: bf16 out[row, n]
// with the activation row taken from sorted_ids (grouped operators).
enum Epi { kGateUp = 0, kDown = 1, kPlain = 2 };

struct StreamParams {
  const uint8_t* tiles;     // blob tile region
  const uint8_t* blob;      // header
  int N, K;                 // physical rows, reduction length
  int E, role;
  const uint16_t* act;      // gate_up: x [T, H]; down: a [cap, I]
  int act_ld;               // elements per activation row (H or I)
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntp;
  int block_m;
  int64_t n_slots;          // T * topk
  int topk;
  int64_t cap;
  uint16_t* out;            // kPlain output [rows, N]
  uint16_t* a_out;          // gate_up output [cap, I]
  float* y_out;             // down output [T*topk, H]
  const float* topk_weights;
  int I, H;
  uint32_t* status;
  float* partial;           // stream-K partial sums [kMaxStreamWorkers][8][32][TC / 2]
  uint32_t* flags;          // stream-K flags [kMaxStreamWorkers][8], zero between launches
};

__device__ __forceinline__ uint4 ldg_nc128(const void* p) {
  uint4 v;
  asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// This warp's code words (rows g and g + 8 of its 16-row block) and scales of one tile.
struct TileCodes {
  uint4 c0, c1, sv;
};
__device__ __forceinline__ TileCodes load_tile_codes(const uint8_t* stg, int tile, int rb, int lane) {
  const uint8_t* st = stg + tile * kTileBytes;
  const int g = lane >> 2, v = g * 16 + code_slot(g, lane & 3) * 4;  // this lane's vector (in words)
  TileCodes tc;
  tc.c0 = *reinterpret_cast<const uint4*>(st + rb * 1024 + v * 4);
  tc.c1 = *reinterpret_cast<const uint4*>(st + rb * 1024 + 512 + v * 4);
  tc.sv = *reinterpret_cast<const uint4*>(st + kTileCodeBytes + rb * 128 + (lane >> 2) * 16);
  return tc;
}

// The activation fragments of one 128-K tile: K step j (32 K) of 8-token tile n8, this
// lane's 8 consecutive K of its token row. xrow[n8] points at the lane's row, already
// offset by 8 * (lane % 4); `off` is the tile's first K.
template <int NT8>
__device__ __forceinline__ void load_tile_x(uint4 (&xv)[4][NT8], const uint16_t* const (&xrow)[NT8], int off) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int n8 = 0; n8 < NT8; ++n8) xv[j][n8] = ldg_nc128(xrow[n8] + off + 32 * j);
}

// Dequantises one tile for warp `rb` (16 rows) and accumulates it against the routed
// activation rows: the A fragments of mma.m16n8k16 come straight out of dequant8; tokens
// are the N dimension. xv holds the tile's activation fragments, loaded at the tile's
// start so that their latency overlaps the first dequantisation. (Refilling each K step's
// fragments with the next tile's right after its MMAs, a whole tile ahead, cut the
// long-scoreboard stalls but measured 3% slower.)
template <int NT8, int NSET>
__device__ __forceinline__ void consume_tile(const TileCodes& code, const uint4 (&xv)[4][NT8],
                                             float (&acc)[NT8][NSET][4], int chain0) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t cw0 = j == 0 ? code.c0.x : j == 1 ? code.c0.y : j == 2 ? code.c0.z : code.c0.w;
    const uint32_t cw1 = j == 0 ? code.c1.x : j == 1 ? code.c1.y : j == 2 ? code.c1.z : code.c1.w;
    // scale pairs: (h0 j0,j1) (h0 j2,j3) (h1 j0,j1) (h1 j2,j3)
    const uint32_t sp0 = (j >> 1) ? code.sv.y : code.sv.x;
    const uint32_t sp1 = (j >> 1) ? code.sv.w : code.sv.z;
    uint32_t w0[4], w1[4];
    dequant8(cw0, bf16_splat_half(sp0, j & 1), w0);
    dequant8(cw1, bf16_splat_half(sp1, j & 1), w1);
    const uint32_t a_lo[4] = {w0[0], w1[0], w0[1], w1[1]};
    const uint32_t a_hi[4] = {w0[2], w1[2], w0[3], w1[3]};
#pragma unroll
    for (int n8 = 0; n8 < NT8; ++n8) {
      mma_bf16_16816(acc[n8][chain0 % NSET], a_lo, xv[j][n8].x, xv[j][n8].y);
      mma_bf16_16816(acc[n8][(chain0 + 1) % NSET], a_hi, xv[j][n8].z, xv[j][n8].w);
    }
  }
}

// The short-K kernel (stream_gemm_short.cu): epi, token columns tc (8, 16 or 32), grid of
// `grid` persistent CTAs; pdl launches it early (programmatic dependent launch).
cudaError_t launch_stream_gemm_short(int epi, const StreamParams& p, int tc, int grid, bool pdl,
                                     cudaStream_t stream);

}  // namespace stream
}  // namespace chord
