// combine.cu -- top-k weighted combine and optional routing validation.
//
// The down kernels write the expert output W2[e] . a of every local flat slot f (by slot
// on the streaming schedule, by sorted position on the tensor-core schedule). The combine
// multiplies each by its top-k weight and sums over the token's local slots in ascending
// slot order in FP32 (acc += w_j * y_j), then rounds once to BF16; a token with no local
// slot gets a zero row.
// The blog excludes this step from its kernel timings ("Messungen"); here it is one
// HBM-bound pass reading T*topk_local*H*4 bytes and writing T*H*2 bytes.
#include "chord_internal.cuh"

namespace chord {
namespace {

constexpr int kCombineThreads = 128;
constexpr int kCombineVecs = 2;                    // 8-output vectors per thread and item
constexpr int kCombineCols = kCombineThreads * 8 * kCombineVecs;  // outputs per work item

// Work item = (token t, 2048 consecutive outputs); a thread owns two vectors of 8 outputs,
// 1024 apart, so each slot's loads come in independent pairs. Lane j % 32
// of every warp holds slot j's weight and row of y (top-k up to 64), and each output
// accumulates its token's local slots in ascending j. BLOCKED selects y by sorted position
// in 128-column blocks [H/128][cap][128] (tensor-core schedule) instead of y by flat slot
// [T*topk, H] (streaming schedule).
// F32OUT writes the FP32 sums (float [T, H]) instead of their BF16 rounding: the partial
// output of one tensor-parallel rank, which the ranks add before the single rounding.
template <bool BLOCKED, bool F32OUT>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const int32_t* __restrict__ topk_ids, const float* __restrict__ topk_weights,
    const float* __restrict__ y, const int32_t* __restrict__ slot_pos, void* __restrict__ out_raw, int64_t T,
    int H, int topk, int E, int64_t cap, const int32_t* __restrict__ ntp, int block_m) {
  grid_dep_wait();  // launched early: y comes from the down kernel
  const int lane = threadIdx.x & 31;
  // routing built for another block_m: the GEMMs computed nothing, so every row is zero
  // (the GEMM kernels raise CHORD_DEV_BLOCK_M_MISMATCH)
  const bool routed = ntp[1] == routing_tag(block_m);
  const int nchunk = (H + kCombineCols - 1) / kCombineCols;
  for (int64_t item = blockIdx.x; item < T * nchunk; item += gridDim.x) {
    const int64_t t = item / nchunk;
    const int c0 = int(item % nchunk) * kCombineCols + threadIdx.x * 8;
    // slot j's row of y (lane j % 32 of set j / 32), or -1 when the slot is not local (or
    // its position is unknown)
    int64_t row[2] = {-1, -1};
    float w[2] = {0.f, 0.f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = h * 32 + lane;
      if (j < topk) {
        const int64_t f = t * topk + j;
        const int e = __ldg(topk_ids + f);
        if (routed && unsigned(e) < unsigned(E)) {
          w[h] = __ldg(topk_weights + f);
          if (BLOCKED) {
            const int pos = __ldg(slot_pos + f);
            row[h] = (pos >= 0 && pos < cap) ? pos : -1;
          } else {
            row[h] = f;
          }
        }
      }
    }
    float acc[kCombineVecs][8];
#pragma unroll
    for (int u = 0; u < kCombineVecs; ++u)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
    // slots in groups of kSlotGroup: the group's rows are all requested before any is
    // summed (one memory round trip per group, not per slot), then added in ascending j
    constexpr int kSlotGroup = 4;
    for (int j0 = 0; j0 < topk; j0 += kSlotGroup) {
      int64_t rj[kSlotGroup];
      float wj[kSlotGroup];
      float4 v[kSlotGroup][kCombineVecs][2];
#pragma unroll
      for (int q = 0; q < kSlotGroup; ++q) {
        const int j = j0 + q;
        rj[q] = -1;
        wj[q] = 0.f;
        if (j < topk) {
          rj[q] = __shfl_sync(0xffffffffu, j < 32 ? row[0] : row[1], j & 31);
          wj[q] = __shfl_sync(0xffffffffu, j < 32 ? w[0] : w[1], j & 31);
        }
#pragma unroll
        for (int u = 0; u < kCombineVecs; ++u) {
          const int c = c0 + u * kCombineThreads * 8;
          v[q][u][0] = v[q][u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (rj[q] >= 0 && c < H) {
            const float* src =
                BLOCKED ? y + ((int64_t(c >> 7) * cap + rj[q]) << 7) + (c & 127) : y + rj[q] * H + c;
            v[q][u][0] = __ldcs(reinterpret_cast<const float4*>(src));
            v[q][u][1] = __ldcs(reinterpret_cast<const float4*>(src) + 1);
          }
        }
      }
      // product rounded, then added (no fused multiply-add), as the layer is defined
#pragma unroll
      for (int q = 0; q < kSlotGroup; ++q) {
        if (rj[q] < 0) continue;
#pragma unroll
        for (int u = 0; u < kCombineVecs; ++u) {
          const float vv[8] = {v[q][u][0].x, v[q][u][0].y, v[q][u][0].z, v[q][u][0].w,
                               v[q][u][1].x, v[q][u][1].y, v[q][u][1].z, v[q][u][1].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[u][i] = __fadd_rn(acc[u][i], __fmul_rn(wj[q], vv[i]));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kCombineVecs; ++u) {
      const int c = c0 + u * kCombineThreads * 8;
      if (c >= H) continue;
      if (F32OUT) {
        float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(out_raw) + t * H + c);
        o4[0] = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
        o4[1] = make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
        continue;
      }
      uint16_t* out = static_cast<uint16_t*>(out_raw);
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[u][2 * i]))) |
               (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[u][2 * i + 1]))) << 16);
      *reinterpret_cast<uint4*>(out + t * H + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Consistency of externally produced routing tensors (CHORD_FLAG_VALIDATE_ROUTING):
// num_tokens_padded is a multiple of block_m within capacity, every used block names a
// local expert, and every entry below num_tokens_padded is padding or a flat slot whose
// topk_ids entry is the block's expert.
__global__ void validate_kernel(const int32_t* __restrict__ topk_ids,
                                const int32_t* __restrict__ sorted_ids,
                                const int32_t* __restrict__ expert_ids,
                                const int32_t* __restrict__ ntp_p, int block_m, int64_t cap,
                                int64_t n_slots, int E, uint32_t* status) {
  // another block_m's routing is reported by the GEMM kernels (CHORD_DEV_BLOCK_M_MISMATCH);
  // its expert_ids may be shorter than this block_m's, so it is not read here
  if (ntp_p[1] != routing_tag(block_m)) return;
  const int ntp = ntp_p[0];
  if (ntp < 0 || ntp > cap || ntp % block_m != 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, CHORD_DEV_ROUTING_INVALID);
    return;
  }
  bool bad = false;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < ntp;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int e = expert_ids[i / block_m];
    const int f = sorted_ids[i];
    if (unsigned(e) >= unsigned(E)) bad = true;
    else if (f < 0) bad = true;
    else if (f < n_slots && topk_ids[f] != e) bad = true;
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, CHORD_DEV_ROUTING_INVALID);
}

}  // namespace

cudaError_t launch_combine(const ForwardArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  int64_t grid = a.T * ((a.H + kCombineCols - 1) / kCombineCols);
  if (grid > int64_t(a.num_sms) * 64) grid = int64_t(a.num_sms) * 64;
  auto kern = a.y_blocked ? (a.out_f32 ? combine_kernel<true, true> : combine_kernel<true, false>)
                          : (a.out_f32 ? combine_kernel<false, true> : combine_kernel<false, false>);
  const cudaError_t err = launch_pdl(a.pdl, kern, dim3(unsigned(grid)), dim3(kCombineThreads), 0, stream, a.topk_ids,
                                     a.topk_weights, static_cast<const float*>(a.y),
                                     static_cast<const int32_t*>(a.slot_pos), static_cast<void*>(a.out), a.T, a.H,
                                     a.topk, a.E, a.cap, a.ntp, a.block_m);
  count_launches(1);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_validate(const ForwardArgs& a, cudaStream_t stream) {
  validate_kernel<<<a.num_sms, 256, 0, stream>>>(a.topk_ids, a.sorted_ids, a.expert_ids, a.ntp,
                                                 a.block_m, a.cap, a.T * a.topk, a.E, a.status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
