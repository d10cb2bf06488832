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
//        chord_ep_pack    the send buffers: hidden rows, local ids, weights
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

// One warp per send row i < num_rows: the token's hidden row, its slots made local to the
// destination rank, and row_of[t * W + d] = i for the combine.
__global__ void __launch_bounds__(256) ep_pack_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_ids,
                                                      const float* __restrict__ topk_weights, int64_t T, int H, int topk,
                                                      int E_rank, int W, const int32_t* __restrict__ send_rows,
                                                      const int32_t* __restrict__ rank_offsets,
                                                      uint16_t* __restrict__ send_x, int32_t* __restrict__ send_ids,
                                                      float* __restrict__ send_w, int32_t* __restrict__ row_of) {
  const int lane = threadIdx.x & 31;
  int64_t rows = rank_offsets[W];
  if (rows < 0) rows = 0;
  if (rows > T * W) rows = T * W;
  const int64_t warp0 = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t i = warp0; i < rows; i += nwarps) {
    const int64_t f = send_rows[i];
    if (f < 0 || f >= T * W) continue;
    const int64_t t = f / W;
    const int d = int(f - t * W);
    if (lane == 0) row_of[f] = int32_t(i);
    for (int j = lane; j < topk; j += 32) {
      const int e = __ldg(topk_ids + t * topk + j);
      const bool here = e >= d * E_rank && e < (d + 1) * E_rank;
      send_ids[i * topk + j] = here ? e - d * E_rank : -1;
      send_w[i * topk + j] = here ? __ldg(topk_weights + t * topk + j) : 0.f;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
    uint4* dst = reinterpret_cast<uint4*>(send_x + i * H);
    for (int v = lane; v < H / 8; v += 32) dst[v] = __ldg(src + v);
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
  ep_pack_kernel<<<grid_for(T * W * 32, 256, num_sms), 256, 0, stream>>>(x, topk_ids, topk_weights, T, H, topk, E_rank,
                                                                         W, send_rows, rank_offsets, send_x, send_ids,
                                                                         send_w, row_of);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const uint16_t* back, const int32_t* row_of, int64_t rows_cap, int64_t T, int H, int W,
                              uint16_t* out, int num_sms, cudaStream_t stream) {
  ep_combine_kernel<<<grid_for(T * (H / 8), 256, num_sms), 256, 0, stream>>>(back, row_of, rows_cap, T, H, W, out);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_round_bf16(const float* in, int64_t n, uint16_t* out, int num_sms, cudaStream_t stream) {
  round_bf16_kernel<<<grid_for(n, 256, num_sms), 256, 0, stream>>>(in, n, out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
