// repack.cu -- one-time weight repack into the tile layout of chord_internal.cuh, and
// the inverse (blob -> logical bf16 weights) used by the layout and dequant checks.
//
// The grouped family of the Chord blog packs a bit-permuted INT4 buffer and re-lays the
// scales once at load, recording the mode in the prepared weight ("Gruppierte
// SM90-Kernel"); this is the sm_100a counterpart: one layout serves both the
// weight-streaming and the tensor-core schedule, so a weight prepared once serves every
// token count (Figure 2: layouts are fixed at model load).
#include "chord_internal.cuh"

namespace chord {
namespace {

__device__ __forceinline__ uint32_t permute_nibbles(uint32_t src) {
  uint32_t out = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) out |= ((src >> (4 * u)) & 0xFu) << (4 * nibble_slot(u));
  return out;
}

// One thread per repacked code word; `tiles` is the blob's tile region.
__global__ void repack_codes_kernel(const int32_t* __restrict__ qweight, int E, int N, int K,
                                    int role, uint8_t* __restrict__ tiles) {
  const int NT = N / kTileN, KT = K / kTileK;
  const int64_t total = int64_t(E) * N * (K / 8);
  for (int64_t w = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; w < total;
       w += int64_t(gridDim.x) * blockDim.x) {
    const int j = int(w & 3), t = int((w >> 2) & 3), g = int((w >> 4) & 7), h = int((w >> 7) & 1);
    const int rb = int((w >> 8) & 7);
    const int64_t tile = w >> 11;
    const int kt = int(tile % KT);
    const int64_t rest = tile / KT;
    const int nt = int(rest % NT);
    const int e = int(rest / NT);
    const int p = nt * kTileN + rb * 16 + 8 * h + g;
    const int n = logical_row(role, N, p);
    const int k0 = kt * kTileK + 32 * j + 8 * t;
    const uint32_t src = uint32_t(qweight[(int64_t(e) * N + n) * (K / 8) + k0 / 8]);
    const int dst = rb * 256 + h * 128 + g * 16 + code_slot(g, t) * 4 + j;
    reinterpret_cast<uint32_t*>(tiles + tile * kTileBytes)[dst] = permute_nibbles(src);
  }
}

// One thread per repacked scale.
__global__ void repack_scales_kernel(const uint16_t* __restrict__ scales, int E, int N, int K,
                                     int role, uint8_t* __restrict__ tiles) {
  const int NT = N / kTileN, KT = K / kTileK;
  const int64_t total = int64_t(E) * N * (K / kGroup);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int j = int(i & 3), h = int((i >> 2) & 1), g = int((i >> 3) & 7), rb = int((i >> 6) & 7);
    const int64_t tile = i >> 9;
    const int kt = int(tile % KT);
    const int64_t rest = tile / KT;
    const int nt = int(rest % NT);
    const int e = int(rest / NT);
    const int p = nt * kTileN + rb * 16 + 8 * h + g;
    const int n = logical_row(role, N, p);
    reinterpret_cast<uint16_t*>(tiles + tile * kTileBytes + kTileCodeBytes)[i & 511] =
        scales[(int64_t(e) * N + n) * (K / kGroup) + kt * 4 + j];
  }
}

__global__ void write_header_kernel(uint8_t* blob, int E, int N, int K, int role) {
  BlobHeader* hd = reinterpret_cast<BlobHeader*>(blob);
  const int i = threadIdx.x;
  if (i < 50) hd->reserved[i] = 0;
  if (i == 0) {
    hd->magic = kBlobMagic;
    hd->version = kBlobVersion;
    hd->layout = kLayoutTile128;
    hd->role = uint32_t(role);
    hd->E = E;
    hd->N = N;
    hd->K = K;
    hd->group = kGroup;
    hd->tiles_offset = blob_tiles_offset();
    hd->tile_bytes = kTileBytes;
    hd->total_bytes = blob_total_bytes(E, N, K);
  }
}

// One thread per repacked word: the same dequant8 the GEMM kernels use, written back
// in logical order w[e][n][k].
__global__ void dequant_blob_kernel(const uint8_t* __restrict__ blob, int E, int N, int K, int role,
                                    uint16_t* __restrict__ w) {
  const int NT = N / kTileN, KT = K / kTileK;
  const uint8_t* tiles = blob + blob_tiles_offset();
  const int64_t total = int64_t(E) * N * (K / 8);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int j = int(i & 3), t = int((i >> 2) & 3), g = int((i >> 4) & 7), h = int((i >> 7) & 1);
    const int rb = int((i >> 8) & 7);
    const int64_t tile = i >> 11;
    const int kt = int(tile % KT);
    const int64_t rest = tile / KT;
    const int nt = int(rest % NT);
    const int e = int(rest / NT);
    const int p = nt * kTileN + rb * 16 + 8 * h + g;
    const int n = logical_row(role, N, p);
    const int k0 = kt * kTileK + 32 * j + 8 * t;
    const uint8_t* tp = tiles + tile * kTileBytes;
    const uint16_t s = reinterpret_cast<const uint16_t*>(tp + kTileCodeBytes)[rb * 64 + g * 8 + h * 4 + j];
    uint32_t pairs[4];
    dequant8(reinterpret_cast<const uint32_t*>(tp)[rb * 256 + h * 128 + g * 16 + code_slot(g, t) * 4 + j],
             bf16_splat(s), pairs);
    uint4 v = make_uint4(pairs[0], pairs[1], pairs[2], pairs[3]);
    *reinterpret_cast<uint4*>(w + (int64_t(e) * N + n) * K + k0) = v;
  }
}

int grid_for(int64_t total, int threads) {
  int64_t g = (total + threads - 1) / threads;
  if (g > 148 * 64) g = 148 * 64;
  return int(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_repack(const int32_t* qweight, const uint16_t* scales, int E, int N, int K,
                          int role, uint8_t* blob, cudaStream_t stream) {
  write_header_kernel<<<1, 64, 0, stream>>>(blob, E, N, K, role);
  const int64_t words = int64_t(E) * N * (K / 8);
  repack_codes_kernel<<<grid_for(words, 256), 256, 0, stream>>>(qweight, E, N, K, role,
                                                                 blob + blob_tiles_offset());
  const int64_t nsc = int64_t(E) * N * (K / kGroup);
  repack_scales_kernel<<<grid_for(nsc, 256), 256, 0, stream>>>(scales, E, N, K, role,
                                                                blob + blob_tiles_offset());
  count_launches(3);
  return cudaGetLastError();
}

cudaError_t launch_dequant_blob(const uint8_t* blob, int E, int N, int K, int role, uint16_t* w,
                                cudaStream_t stream) {
  const int64_t words = int64_t(E) * N * (K / 8);
  dequant_blob_kernel<<<grid_for(words, 256), 256, 0, stream>>>(blob, E, N, K, role, w);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
