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
constexpr int kCombineVecs = 4;                    // 8-output vectors per lane and unit
constexpr int kUnitCols = 32 * 8 * kCombineVecs;   // outputs per unit (one warp)
constexpr int kSlotGroup = 2;                      // local slots whose rows are loaded together

// A token's slots as one warp sees them: lane j % 32 of half j / 32 holds slot j's row
// of y (-1 when the slot is not local or its position is unknown) and top-k weight.
struct SlotRows {
  int row[2];  // < 2^31: the routing capacity and T*topk are checked below that
  float w[2];
};

// Issues every load of token t's slot metadata at once (ids, weights and positions do
// not depend on one another), so a prefetch of the next unit's token overlaps the current
// unit's rows of y.
template <bool BLOCKED>
__device__ __forceinline__ void load_slot_rows(SlotRows& m, int64_t t, int lane, const int32_t* __restrict__ topk_ids,
                                               const float* __restrict__ topk_weights,
                                               const int32_t* __restrict__ slot_pos, int topk, int E, int64_t cap,
                                               bool routed) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = h * 32 + lane;
    m.row[h] = -1;
    m.w[h] = 0.f;
    if (j < topk) {
      const int64_t f = t * topk + j;
      const int e = __ldg(topk_ids + f);
      const float w = __ldg(topk_weights + f);
      const int pos = BLOCKED ? __ldg(slot_pos + f) : 0;
      if (routed && unsigned(e) < unsigned(E)) {
        m.w[h] = w;
        m.row[h] = BLOCKED ? ((pos >= 0 && pos < cap) ? pos : -1) : int(f);
      }
    }
  }
}

// Unit = (token t, kUnitCols consecutive outputs), one warp; a lane owns kCombineVecs
// vectors of 8 outputs, 256 apart, so a warp's loads and stores of one vector index are
// contiguous. The token's local slots are found with one ballot and taken in ascending j,
// kSlotGroup at a time: the group's rows are all requested before any is summed, and slots
// that are not local cost nothing. Each output accumulates w_j * y_j in ascending j in
// FP32 (product rounded, then added). Warps walk units with a grid stride and load the
// next unit's slot metadata before summing the current one, so a unit costs one memory
// round trip per slot group.
// BLOCKED selects y by sorted position in 128-column blocks [H/128][cap][128] (tensor-core
// schedule) instead of y by flat slot [T*topk, H] (streaming schedule). F32OUT writes the
// FP32 sums (float [T, H]) instead of their BF16 rounding: the partial output of one
// tensor-parallel rank, which the ranks add before the single rounding.
template <bool BLOCKED, bool F32OUT>
__global__ void __launch_bounds__(kCombineThreads, 4) combine_kernel(
    const int32_t* __restrict__ topk_ids, const float* __restrict__ topk_weights,
    const float* __restrict__ y, const int32_t* __restrict__ slot_pos, void* __restrict__ out_raw, int64_t T,
    int H, int topk, int E, int64_t cap, const int32_t* __restrict__ ntp, int block_m) {
  grid_dep_wait();  // launched early: y comes from the down kernel
  const int lane = threadIdx.x & 31;
  // routing built for another block_m: the GEMMs computed nothing, so every row is zero
  // (the GEMM kernels raise CHORD_DEV_BLOCK_M_MISMATCH)
  const bool routed = ntp[1] == routing_tag(block_m);
  const int nseg = (H + kUnitCols - 1) / kUnitCols;
  const int64_t units = T * nseg;
  const int64_t nwarps = (int64_t(gridDim.x) * kCombineThreads) >> 5;
  int64_t u = (int64_t(blockIdx.x) * kCombineThreads + threadIdx.x) >> 5;
  if (u >= units) return;
  SlotRows cur;
  int64_t t = u / nseg;
  load_slot_rows<BLOCKED>(cur, t, lane, topk_ids, topk_weights, slot_pos, topk, E, cap, routed);
  for (; u < units; u += nwarps) {
    const int seg = int(u - t * nseg);
    // the next unit's token: its metadata loads go out now
    const int64_t un = u + nwarps;
    const int64_t tn = un < units ? un / nseg : t;
    SlotRows nxt = cur;
    if (tn != t) load_slot_rows<BLOCKED>(nxt, tn, lane, topk_ids, topk_weights, slot_pos, topk, E, cap, routed);

    const int c0 = seg * kUnitCols + lane * 8;
    float acc[kCombineVecs][8];
#pragma unroll
    for (int k = 0; k < kCombineVecs; ++k)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[k][i] = 0.f;
    // local slots, ascending j (warp-uniform masks)
    uint32_t mask0 = __ballot_sync(0xffffffffu, cur.row[0] >= 0);
    uint32_t mask1 = topk > 32 ? __ballot_sync(0xffffffffu, cur.row[1] >= 0) : 0u;
    while (mask0 | mask1) {
      int rj[kSlotGroup];
      float wj[kSlotGroup];
      float4 v[kSlotGroup][kCombineVecs][2];
#pragma unroll
      for (int q = 0; q < kSlotGroup; ++q) {
        rj[q] = -1;
        wj[q] = 0.f;
        if (mask0) {
          const int src = __ffs(mask0) - 1;
          mask0 &= mask0 - 1;
          rj[q] = __shfl_sync(0xffffffffu, cur.row[0], src);
          wj[q] = __shfl_sync(0xffffffffu, cur.w[0], src);
        } else if (mask1) {
          const int src = __ffs(mask1) - 1;
          mask1 &= mask1 - 1;
          rj[q] = __shfl_sync(0xffffffffu, cur.row[1], src);
          wj[q] = __shfl_sync(0xffffffffu, cur.w[1], src);
        }
#pragma unroll
        for (int k = 0; k < kCombineVecs; ++k) {
          const int c = c0 + k * 256;
          v[q][k][0] = v[q][k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (rj[q] >= 0 && c < H) {
            const float* src =
                BLOCKED ? y + ((int64_t(c >> 7) * cap + rj[q]) << 7) + (c & 127) : y + int64_t(rj[q]) * H + c;
            v[q][k][0] = __ldcs(reinterpret_cast<const float4*>(src));
            v[q][k][1] = __ldcs(reinterpret_cast<const float4*>(src) + 1);
          }
        }
      }
      // product rounded, then added (no fused multiply-add), as the layer is defined
#pragma unroll
      for (int q = 0; q < kSlotGroup; ++q) {
        if (rj[q] < 0) continue;
#pragma unroll
        for (int k = 0; k < kCombineVecs; ++k) {
          const float vv[8] = {v[q][k][0].x, v[q][k][0].y, v[q][k][0].z, v[q][k][0].w,
                               v[q][k][1].x, v[q][k][1].y, v[q][k][1].z, v[q][k][1].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[k][i] = __fadd_rn(acc[k][i], __fmul_rn(wj[q], vv[i]));
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kCombineVecs; ++k) {
      const int c = c0 + k * 256;
      if (c >= H) continue;
      if (F32OUT) {
        float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(out_raw) + t * H + c);
        o4[0] = make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
        o4[1] = make_float4(acc[k][4], acc[k][5], acc[k][6], acc[k][7]);
        continue;
      }
      uint16_t* out = static_cast<uint16_t*>(out_raw);
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[k][2 * i]))) |
               (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[k][2 * i + 1]))) << 16);
      *reinterpret_cast<uint4*>(out + t * H + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    cur = nxt;
    t = tn;
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
  // one unit per warp, warps resident all at once (4 CTAs per SM by the launch bounds):
  // each walks its units with the next unit's metadata in flight
  const int64_t units = a.T * ((a.H + kUnitCols - 1) / kUnitCols);
  int64_t grid = (units + kCombineThreads / 32 - 1) / (kCombineThreads / 32);
  if (grid > int64_t(a.num_sms) * 4) grid = int64_t(a.num_sms) * 4;
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
