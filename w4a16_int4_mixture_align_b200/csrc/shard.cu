// shard.cu -- the exchange steps around the layer when it is sharded over several GPUs.
//
// The Chord blog deploys the layer as expert-parallel (EP8/EP16/EP32) and tensor-parallel
// (TP8) shards ("TL;DR"; "vLLM-Integration": the TP8 single-instance profile) and times
// the kernels without the communication ("Messungen"). The exchanges themselves are:
//
//  EP: each rank owns E_rank consecutive global experts. A token is sent once to every
//      rank that owns at least one of its top-k experts, with the slot ids made local to
//      that rank (-1 for slots owned elsewhere) and the matching top-k weights (0
//      elsewhere); each rank runs the layer on what it received, returns one output row per
//      received row, and the source sums a token's returned rows.
//        chord_ep_plan    send rows grouped by destination rank, ascending token inside
//                         each (the routing sort of the layer over W "experts" = ranks)
//        chord_ep_pack    row_of (the inverse of send_rows), then the send buffers token by
//                         token: each piece of a hidden row read once and stored into each
//                         of its send rows, with the local ids and weights
//        chord_ep_combine out[t] = bf16( sum over ranks d, ascending, of float(back row) )
//  TP: each rank owns a slice of the intermediate dimension of every expert; its layer
//      output is a partial sum of the full layer's FP32 result. chord_moe_forward with
//      CHORD_FLAG_OUTPUT_FP32 keeps those sums in FP32, the ranks all-reduce them, and
//      chord_round_bf16 rounds the total once.
//
// The collectives between these steps (all-to-all, all-reduce) are the caller's: NCCL
// through torch.distributed in the Python binding.
#include "chord_internal.cuh"

namespace chord {
namespace {

// ids_tw[t * W + d] = d when token t has a slot on rank d, else -1; row_of = -1 everywhere
__global__ void __launch_bounds__(256) ep_route_kernel(const int32_t* __restrict__ topk_ids, int64_t T, int topk,
                                                       int E_rank, int W, int32_t* __restrict__ ids_tw,
                                                       int32_t* __restrict__ row_of) {
  const int64_t n = T * W;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / W;
    const int d = int(i - t * W);
    int hit = -1;
    for (int j = 0; j < topk; ++j) {
      const int e = __ldg(topk_ids + t * topk + j);
      if (e >= d * E_rank && e < (d + 1) * E_rank) hit = d;
    }
    ids_tw[i] = hit;
    row_of[i] = -1;
  }
}

// row_of[send_rows[i]] = i for every send row i < rank_offsets[W] (the other entries stay
// -1 from the route kernel): the send row of each (token, rank) pair.
__global__ void __launch_bounds__(256) ep_invert_kernel(const int32_t* __restrict__ send_rows,
                                                        const int32_t* __restrict__ rank_offsets, int64_t T, int W,
                                                        int32_t* __restrict__ row_of) {
  int64_t rows = rank_offsets[W];
  if (rows < 0) rows = 0;
  if (rows > T * W) rows = T * W;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < rows; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t f = send_rows[i];
    if (f >= 0 && f < T * W) row_of[f] = int32_t(i);
  }
}

// One warp per (token t, 1024-column chunk), token-major: the token's send rows
// (row_of[t*W + d], lane d % 32 of half d / 32) are found with a ballot; each 16-byte vector
// of the chunk is read once (four per lane) and stored into every one of them, so a row
// sent to several ranks is read from memory once, and a small batch still spreads over
// many warps. The chunk-0 warp also writes each send row's slots made local to its rank
// (-1 elsewhere) and their weights (0 elsewhere).
constexpr int kPackVecs = 4;                    // 16-byte vectors per lane and chunk
constexpr int kPackChunk = 32 * kPackVecs;      // vectors per chunk (1024 bf16 columns)

__global__ void __launch_bounds__(256) ep_pack_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_ids,
                                                      const float* __restrict__ topk_weights, int64_t T, int H, int topk,
                                                      int E_rank, int W, const int32_t* __restrict__ row_of,
                                                      uint16_t* __restrict__ send_x, int32_t* __restrict__ send_ids,
                                                      float* __restrict__ send_w) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t cap = T * W;
  const int nvec = H / 8;
  const int nchunk = (nvec + kPackChunk - 1) / kPackChunk;
  for (int64_t unit = warp0; unit < T * nchunk; unit += nwarps) {
    const int64_t t = unit / nchunk;
    const int chunk = int(unit - t * nchunk);
    int i0 = lane < W ? __ldg(row_of + t * W + lane) : -1;
    int i1 = lane + 32 < W ? __ldg(row_of + t * W + lane + 32) : -1;
    if (i0 >= cap) i0 = -1;
    if (i1 >= cap) i1 = -1;
    const uint32_t m0 = __ballot_sync(0xffffffffu, i0 >= 0), m1 = __ballot_sync(0xffffffffu, i1 >= 0);
    if ((m0 | m1) == 0) continue;
    const int v0 = chunk * kPackChunk + lane;
    uint4 val[kPackVecs];
    const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
#pragma unroll
    for (int u = 0; u < kPackVecs; ++u)
      if (v0 + 32 * u < nvec) val[u] = __ldg(src + v0 + 32 * u);
    for (int h = 0; h < 2; ++h) {
      uint32_t m = h ? m1 : m0;
      while (m) {
        const int dl = __ffs(m) - 1;
        m &= m - 1;
        const int d = h * 32 + dl;
        const int i = __shfl_sync(0xffffffffu, h ? i1 : i0, dl);
        uint4* dst = reinterpret_cast<uint4*>(send_x + int64_t(i) * H);
#pragma unroll
        for (int u = 0; u < kPackVecs; ++u)
          if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = val[u];
        if (chunk == 0) {
          for (int j = lane; j < topk; j += 32) {
            const int e = __ldg(topk_ids + t * topk + j);
            const bool here = e >= d * E_rank && e < (d + 1) * E_rank;
            send_ids[int64_t(i) * topk + j] = here ? e - d * E_rank : -1;
            send_w[int64_t(i) * topk + j] = here ? __ldg(topk_weights + t * topk + j) : 0.f;
          }
        }
      }
    }
  }
}

// out[t, c] = bf16( sum over d = 0 .. W-1 with a row of float(back[row_of[t*W+d], c]) ),
// eight outputs per thread; 0 for a token that sent nothing.
__global__ void __launch_bounds__(256) ep_combine_kernel(const uint16_t* __restrict__ back,
                                                         const int32_t* __restrict__ row_of, int64_t rows_cap,
                                                         int64_t T, int H, int W, uint16_t* __restrict__ out) {
  const int nv = H / 8;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < T * nv; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / nv;
    const int c = int(i - t * nv) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int d = 0; d < W; ++d) {
      const int r = __ldg(row_of + t * W + d);
      if (r < 0 || r >= rows_cap) continue;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(back + int64_t(r) * H + c));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] = __fadd_rn(acc[2 * k], __uint_as_float(w[k] << 16));
        acc[2 * k + 1] = __fadd_rn(acc[2 * k + 1], __uint_as_float(w[k] & 0xFFFF0000u));
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      o[k] = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * k]))) |
             (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * k + 1]))) << 16);
    *reinterpret_cast<uint4*>(out + t * H + c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__global__ void __launch_bounds__(256) round_bf16_kernel(const float* __restrict__ in, int64_t n,
                                                         uint16_t* __restrict__ out) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(in[i]));
}

// Tensor-parallel reduction over the ranks' buffers by pointer (peer memory, or one GPU's
// own buffers standing in for the ranks): this rank's slice [v0, v1) of the 4-float
// vectors, out[d][i] = bf16( sum over s = 0 .. W-1, ascending, of partials[s][i] ) stored
// into every rank d's output. Every rank sums in the same order, so all outputs agree bit
// for bit.
__global__ void __launch_bounds__(256) tp_reduce_round_kernel(TpPeers peers, int W, int64_t v0, int64_t v1) {
  for (int64_t v = v0 + int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < v1; v += int64_t(gridDim.x) * blockDim.x) {
    float4 acc = __ldcg(reinterpret_cast<const float4*>(peers.in[0]) + v);
    for (int s = 1; s < W; ++s) {
      const float4 x = __ldcg(reinterpret_cast<const float4*>(peers.in[s]) + v);
      acc.x = __fadd_rn(acc.x, x.x);
      acc.y = __fadd_rn(acc.y, x.y);
      acc.z = __fadd_rn(acc.z, x.z);
      acc.w = __fadd_rn(acc.w, x.w);
    }
    const uint2 o = make_uint2(uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.x))) |
                                   (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.y))) << 16),
                               uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.z))) |
                                   (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.w))) << 16));
    for (int d = 0; d < W; ++d) reinterpret_cast<uint2*>(peers.out[d])[v] = o;
  }
}

unsigned grid_for(int64_t n, int threads, int num_sms) {
  int64_t g = (n + threads - 1) / threads;
  const int64_t cap = int64_t(num_sms) * 16;
  if (g > cap) g = cap;
  return unsigned(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_ep_route(const int32_t* topk_ids, int64_t T, int topk, int E_rank, int W, int32_t* ids_tw,
                            int32_t* row_of, int num_sms, cudaStream_t stream) {
  ep_route_kernel<<<grid_for(T * W, 256, num_sms), 256, 0, stream>>>(topk_ids, T, topk, E_rank, W, ids_tw, row_of);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_ep_pack(const uint16_t* x, const int32_t* topk_ids, const float* topk_weights, int64_t T, int H,
                           int topk, int E_rank, int W, const int32_t* send_rows, const int32_t* rank_offsets,
                           uint16_t* send_x, int32_t* send_ids, float* send_w, int32_t* row_of, int num_sms,
                           cudaStream_t stream) {
  ep_invert_kernel<<<grid_for(T * W, 256, num_sms), 256, 0, stream>>>(send_rows, rank_offsets, T, W, row_of);
  const int64_t units = T * ((H / 8 + kPackChunk - 1) / kPackChunk);
  ep_pack_kernel<<<grid_for(units * 32, 256, num_sms), 256, 0, stream>>>(x, topk_ids, topk_weights, T, H, topk, E_rank,
                                                                         W, row_of, send_x, send_ids, send_w);
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const uint16_t* back, const int32_t* row_of, int64_t rows_cap, int64_t T, int H, int W,
                              uint16_t* out, int num_sms, cudaStream_t stream) {
  ep_combine_kernel<<<grid_for(T * (H / 8), 256, num_sms), 256, 0, stream>>>(back, row_of, rows_cap, T, H, W, out);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tp_reduce_round(const TpPeers& peers, int W, int rank, int64_t n, int num_sms, cudaStream_t stream) {
  const int64_t nv = n / 4;
  const int64_t v0 = nv * rank / W, v1 = nv * (rank + 1) / W;
  if (v1 <= v0) return cudaSuccess;
  tp_reduce_round_kernel<<<grid_for(v1 - v0, 256, num_sms), 256, 0, stream>>>(peers, W, v0, v1);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_round_bf16(const float* in, int64_t n, uint16_t* out, int num_sms, cudaStream_t stream) {
  round_bf16_kernel<<<grid_for(n, 256, num_sms), 256, 0, stream>>>(in, n, out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
