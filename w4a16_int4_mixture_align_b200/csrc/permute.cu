// permute.cu -- hidden rows into routing order for the tensor-core schedule.
//
// The tensor-core GEMMs read the activation operand as whole tiles of consecutive rows
// (one TMA box per 128-K step), so the hidden states are copied once into the order of
// sorted_ids (the routing sort of the Chord blog's indexed path), row-major:
// xs[pos][c] = x[sorted_ids[pos] / topk][c]. Padding positions (sentinel slots) are not
// written; the GEMMs never read them back into a result.
//
// Two passes: slot_pos[f] = pos, the inverse of sorted_ids over the local slots (with
// which the combine also finds a slot's expert output in the position-ordered y); then the
// copy, token by token, so that a hidden row routed to several experts (a TP8 token to
// eight) is read from memory once and stored at each of its positions. The reads ask L2 to
// keep the rows (evict_last) while the copies, larger than L2, stream out (evict_first).
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

// slot_pos[f] = pos for every routed position (the inverse of sorted_ids over the local
// slots); padding positions are skipped.
__global__ void __launch_bounds__(256) slot_positions_kernel(const int32_t* __restrict__ sorted_ids,
                                                             const int32_t* __restrict__ ntp_p, int block_m,
                                                             int64_t cap, int64_t n_slots,
                                                             int32_t* __restrict__ slot_pos,
                                                             uint32_t* __restrict__ status) {
  const int64_t ntp = routed_positions(ntp_p, block_m, cap, status);
  for (int64_t pos = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; pos < ntp;
       pos += int64_t(gridDim.x) * blockDim.x) {
    const int f = __ldg(sorted_ids + pos);
    if (f >= 0 && f < n_slots) slot_pos[f] = int32_t(pos);
  }
}

// One warp per (token t, 1024-column piece), token-major: the piece of t's hidden row is
// read once (four 16-byte vectors per lane) and stored at the sorted position of each of
// t's local slots (lane j holds slot j's position; found with a ballot), so a row routed
// to several experts is read from memory once.
constexpr int kPermuteVecs = 4;
constexpr int kPermuteChunk = 32 * kPermuteVecs;  // 16-byte vectors per piece

__global__ void __launch_bounds__(32 * kPermuteWarps) permute_rows_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_ids, const int32_t* __restrict__ ntp_p,
    int block_m, int64_t cap, int64_t T, int topk, int E, int H, const int32_t* __restrict__ slot_pos,
    uint16_t* __restrict__ xs) {
  const int lane = threadIdx.x & 31;
  // routing built for another block_m: the GEMMs read nothing of xs
  if (ntp_p[1] != routing_tag(block_m)) return;
  const int64_t warp0 = int64_t(blockIdx.x) * kPermuteWarps + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * kPermuteWarps;
  const int nvec = H / 8;
  const int nchunk = (nvec + kPermuteChunk - 1) / kPermuteChunk;
  const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
  for (int64_t unit = warp0; unit < T * nchunk; unit += nwarps) {
    const int64_t t = unit / nchunk;
    const int chunk = int(unit - t * nchunk);
    int p0 = -1, p1 = -1;  // slot lane's (and lane + 32's) sorted position, -1 when not local
    if (lane < topk) {
      const int e = __ldg(topk_ids + t * topk + lane);
      if (unsigned(e) < unsigned(E)) p0 = __ldg(slot_pos + t * topk + lane);
    }
    if (lane + 32 < topk) {
      const int e = __ldg(topk_ids + t * topk + lane + 32);
      if (unsigned(e) < unsigned(E)) p1 = __ldg(slot_pos + t * topk + lane + 32);
    }
    if (p0 >= cap) p0 = -1;
    if (p1 >= cap) p1 = -1;
    const uint32_t m0 = __ballot_sync(0xffffffffu, p0 >= 0), m1 = __ballot_sync(0xffffffffu, p1 >= 0);
    if ((m0 | m1) == 0) continue;
    const int v0 = chunk * kPermuteChunk + lane;
    const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
    uint4 val[kPermuteVecs];
#pragma unroll
    for (int u = 0; u < kPermuteVecs; ++u)
      if (v0 + 32 * u < nvec) val[u] = ldg_keep(src + v0 + 32 * u, keep);
    for (int h = 0; h < 2; ++h) {
      uint32_t m = h ? m1 : m0;
      while (m) {
        const int sl = __ffs(m) - 1;
        m &= m - 1;
        const int pos = __shfl_sync(0xffffffffu, h ? p1 : p0, sl);
        uint4* dst = reinterpret_cast<uint4*>(xs + int64_t(pos) * H);
#pragma unroll
        for (int u = 0; u < kPermuteVecs; ++u)
          if (v0 + 32 * u < nvec) stg_stream(dst + v0 + 32 * u, val[u], stream);
      }
    }
  }
}

}  // namespace

cudaError_t launch_permute_rows(const ForwardArgs& a, cudaStream_t stream) {
  int64_t ctas = (a.cap + 255) / 256;
  if (ctas > int64_t(a.num_sms) * 8) ctas = int64_t(a.num_sms) * 8;
  if (ctas < 1) ctas = 1;
  slot_positions_kernel<<<unsigned(ctas), 256, 0, stream>>>(a.sorted_ids, a.ntp, a.block_m, a.cap, a.T * a.topk,
                                                            a.slot_pos, a.status);
  const int64_t units = a.T * ((a.H / 8 + kPermuteChunk - 1) / kPermuteChunk);
  int64_t pctas = (units + kPermuteWarps - 1) / kPermuteWarps;
  if (pctas > int64_t(a.num_sms) * 8) pctas = int64_t(a.num_sms) * 8;
  if (pctas < 1) pctas = 1;
  permute_rows_kernel<<<unsigned(pctas), 32 * kPermuteWarps, 0, stream>>>(a.x, a.topk_ids, a.ntp, a.block_m, a.cap,
                                                                          a.T, a.topk, a.E, a.H, a.slot_pos, a.xs);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace chord
