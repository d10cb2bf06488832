// combine.cu -- top-k weighted combine and optional routing validation.
//
// The down kernels write y[f, :] = W2[e] . a for every local flat slot f. The combine
// multiplies each row by its top-k weight and sums over the token's local slots in
// ascending slot order in FP32 (acc += w_j * y_j), then rounds once to BF16; a token with
// no local slot gets a zero row.
// The blog excludes this step from its kernel timings ("Messungen"); here it is one
// HBM-bound pass reading T*topk_local*H*4 bytes and writing T*H*2 bytes.
#include "chord_internal.cuh"

namespace chord {
namespace {

// One thread per 8 consecutive outputs of one token.
__global__ void __launch_bounds__(256) combine_kernel(const int32_t* __restrict__ topk_ids,
                                                      const float* __restrict__ topk_weights,
                                                      const float* __restrict__ y,
                                                      uint16_t* __restrict__ out, int64_t T,
                                                      int H, int topk, int E) {
  const int vec_per_row = H / 8;
  const int64_t total = T * vec_per_row;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i / vec_per_row;
    const int c = int(i % vec_per_row) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < topk; ++j) {
      const int e = __ldg(topk_ids + t * topk + j);
      if (unsigned(e) >= unsigned(E)) continue;
      const float w = __ldg(topk_weights + t * topk + j);
      const float4* src = reinterpret_cast<const float4*>(y + (t * topk + j) * int64_t(H) + c);
      const float4 v0 = __ldcs(src), v1 = __ldcs(src + 1);
      // product rounded, then added (no fused multiply-add), as the layer is defined
      acc[0] = __fadd_rn(acc[0], __fmul_rn(w, v0.x)); acc[1] = __fadd_rn(acc[1], __fmul_rn(w, v0.y));
      acc[2] = __fadd_rn(acc[2], __fmul_rn(w, v0.z)); acc[3] = __fadd_rn(acc[3], __fmul_rn(w, v0.w));
      acc[4] = __fadd_rn(acc[4], __fmul_rn(w, v1.x)); acc[5] = __fadd_rn(acc[5], __fmul_rn(w, v1.y));
      acc[6] = __fadd_rn(acc[6], __fmul_rn(w, v1.z)); acc[7] = __fadd_rn(acc[7], __fmul_rn(w, v1.w));
    }
    uint4 o;
    o.x = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[0]))) |
          (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[1]))) << 16);
    o.y = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2]))) |
          (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[3]))) << 16);
    o.z = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[4]))) |
          (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[5]))) << 16);
    o.w = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[6]))) |
          (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc[7]))) << 16);
    *reinterpret_cast<uint4*>(out + t * H + c) = o;
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
  const int ntp = *ntp_p;
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
  const int64_t total = a.T * (a.H / 8);
  if (total == 0) return cudaSuccess;
  int64_t grid = (total + 255) / 256;
  if (grid > int64_t(a.num_sms) * 16) grid = int64_t(a.num_sms) * 16;
  combine_kernel<<<unsigned(grid), 256, 0, stream>>>(a.topk_ids, a.topk_weights, a.y, a.out, a.T, a.H,
                                                      a.topk, a.E);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_validate(const ForwardArgs& a, cudaStream_t stream) {
  validate_kernel<<<a.num_sms, 256, 0, stream>>>(a.topk_ids, a.sorted_ids, a.expert_ids, a.ntp,
                                                 a.block_m, a.cap, a.T * a.topk, a.E, a.status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
