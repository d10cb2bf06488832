// permute.cu -- hidden rows into routing order for the tensor-core schedule.
//
// The tensor-core GEMMs read the activation operand as whole tiles of consecutive rows
// (one TMA box per 128-K step), so the hidden states are copied once into the order of
// sorted_ids (the routing sort of the Chord blog's indexed path), row-major:
// xs[pos][c] = x[sorted_ids[pos] / topk][c]. Padding positions (sentinel slots) are
// skipped; the GEMMs never read them back into a result.
// The same pass records slot_pos[f] = pos, the inverse of sorted_ids over the local
// slots, with which the combine finds a slot's expert output in the position-ordered y.
//
// One warp copies one routed row, 512 contiguous bytes per step each way. A hidden row is
// read once per local slot of its token (up to top-k times), so the reads ask L2 to keep
// it (evict_last) while the copies, larger than L2, stream out (evict_first).
#include "chord_internal.cuh"

namespace chord {
namespace {

constexpr int kPermuteWarps = 8;

__device__ __forceinline__ uint4 ldg_keep(const void* p, uint64_t pol) {
  uint4 v;
  asm("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ void stg_stream(void* p, const uint4& v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w), "l"(pol)
               : "memory");
}

__global__ void __launch_bounds__(32 * kPermuteWarps) permute_rows_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_ids, const int32_t* __restrict__ ntp_p,
    int block_m, int64_t cap, int64_t n_slots, int topk, int H, uint16_t* __restrict__ xs,
    int32_t* __restrict__ slot_pos, uint32_t* __restrict__ status) {
  const int64_t ntp = routed_positions(ntp_p, block_m, cap, status);
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = int64_t(blockIdx.x) * kPermuteWarps + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * kPermuteWarps;
  const int vec = H / 8;  // 16-byte vectors per row
  const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
  for (int64_t pos = warp0; pos < ntp; pos += nwarps) {
    const int f = __ldg(sorted_ids + pos);
    if (f < 0 || f >= n_slots) continue;
    if (lane == 0) slot_pos[f] = int32_t(pos);
    const uint4* src = reinterpret_cast<const uint4*>(x + int64_t(f / topk) * H);
    uint4* dst = reinterpret_cast<uint4*>(xs + pos * H);
    // four 16-byte loads in flight per lane before their stores: with one, the copy ran at
    // about half the HBM write rate when the hidden rows come from L2 (TP8 prefill)
    constexpr int U = 4;
    for (int v0 = lane; v0 < vec; v0 += 32 * U) {
      uint4 t[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (v0 + 32 * u < vec) t[u] = ldg_keep(src + v0 + 32 * u, keep);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (v0 + 32 * u < vec) stg_stream(dst + v0 + 32 * u, t[u], stream);
    }
  }
}

}  // namespace

cudaError_t launch_permute_rows(const ForwardArgs& a, cudaStream_t stream) {
  int64_t ctas = (a.cap + kPermuteWarps - 1) / kPermuteWarps;
  if (ctas > int64_t(a.num_sms) * 8) ctas = int64_t(a.num_sms) * 8;
  if (ctas < 1) ctas = 1;
  permute_rows_kernel<<<unsigned(ctas), 32 * kPermuteWarps, 0, stream>>>(a.x, a.sorted_ids, a.ntp, a.block_m, a.cap,
                                                                         a.T * a.topk, a.topk, a.H, a.xs,
                                                                         a.slot_pos, a.status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
