// permute.cu -- hidden rows into routing order for the tensor-core schedule.
//
// The tensor-core GEMMs read the activation operand as whole tiles of consecutive rows
// (one TMA box per 128-K step), so the hidden states are copied once into the order of
// sorted_ids (the routing sort of the Chord blog's indexed path), K-blocked as
// [H/64][cap][64]: xs[c / 64][pos][c % 64] = x[sorted_ids[pos] / topk][c]. Padding
// positions (sentinel slots) are skipped; the GEMMs never read them back into a result.
//
// One warp copies one routed row: 32 lanes read 512 contiguous bytes of the source row
// per step and write them as four 128-byte runs, one per 64-column chunk.
#include "chord_internal.cuh"

namespace chord {
namespace {

constexpr int kPermuteWarps = 8;

__global__ void __launch_bounds__(32 * kPermuteWarps) permute_rows_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ sorted_ids, const int32_t* __restrict__ ntp_p,
    int64_t cap, int64_t n_slots, int topk, int H, uint16_t* __restrict__ xs) {
  int64_t ntp = *ntp_p;
  if (ntp < 0) ntp = 0;
  if (ntp > cap) ntp = cap;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = int64_t(blockIdx.x) * kPermuteWarps + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * kPermuteWarps;
  const int vec = H / 8;  // 16-byte vectors per row
  for (int64_t pos = warp0; pos < ntp; pos += nwarps) {
    const int f = __ldg(sorted_ids + pos);
    if (f < 0 || f >= n_slots) continue;
    const uint4* src = reinterpret_cast<const uint4*>(x + int64_t(f / topk) * H);
    uint16_t* dst = xs + pos * 64;
    for (int v = lane; v < vec; v += 32) {
      const uint4 val = __ldg(src + v);
      const int c = v * 8;
      *reinterpret_cast<uint4*>(dst + int64_t(c >> 6) * cap * 64 + (c & 63)) = val;
    }
  }
}

}  // namespace

cudaError_t launch_permute_rows(const ForwardArgs& a, cudaStream_t stream) {
  int64_t ctas = (a.cap + kPermuteWarps - 1) / kPermuteWarps;
  if (ctas > int64_t(a.num_sms) * 8) ctas = int64_t(a.num_sms) * 8;
  if (ctas < 1) ctas = 1;
  permute_rows_kernel<<<unsigned(ctas), 32 * kPermuteWarps, 0, stream>>>(a.x, a.sorted_ids, a.ntp, a.cap,
                                                                         a.T * a.topk, a.topk, a.H, a.xs);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
