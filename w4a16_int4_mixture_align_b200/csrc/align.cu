// align.cu -- block-padded routing sort (moe_align) for sm_100a.
//
// The indexed W4A16 path consumes vLLM-style sorted routing: sorted_ids / expert_ids /
// num_tokens_padded, with the activations left unpadded and padding carried by
// sentinel indices (Chord blog, "Zwei Kernel-Familien" and Figure 3). This file builds
// those tensors deterministically: inside each expert the flat slot indices appear in
// increasing order, so the result is a function of topk_ids alone.
//
// Work split: a warp owns a run of consecutive 32-slot steps. Inside a step, the lanes
// holding the same expert are found with one ballot per key bit; a lane's rank is the
// popcount of its lower peers, and the lowest peer advances the expert's running
// position. Runs are ordered by a prefix over per-run histograms.
//
//   n <= 4 x 1024  : one CTA of 32 warps (runs of ceil(n/1024) steps) does count, scan,
//                    scatter and fill (1 launch)
//   larger n       : count kernel (per-chunk histograms) -> scan kernel (1 CTA) ->
//                    scatter + fill kernel, histograms in the caller's workspace.
#include "chord_internal.cuh"

namespace chord {
namespace {

constexpr int kChunk = 1024;       // flat slots per warp chunk
constexpr int kSteps = kChunk / 32;
constexpr int kMaxE = 1024;
// Up to this many 1024-slot chunks the routing sort runs in one CTA (one launch); above
// it the count / scan / scatter kernels spread the slots over the GPU (one CTA sorting
// 32 chunks took ~70 us).
constexpr int kSingleMaxChunks = 4;

__device__ __forceinline__ bool is_local(int e, int E) { return unsigned(e) < unsigned(E); }

// Lanes of the warp holding the same key as this lane (key < 2^nbits), from one ballot
// per key bit: cheaper than __match_any_sync when a step holds many distinct keys.
__device__ __forceinline__ unsigned peers_of(unsigned key, int nbits) {
  unsigned eq = 0xffffffffu;
  for (int b = 0; b < nbits; ++b) {
    const unsigned bit = (key >> b) & 1u;
    const unsigned m = __ballot_sync(0xffffffffu, bit);
    eq &= bit ? m : ~m;
  }
  return eq;
}

__host__ __device__ inline int key_bits(int E) {
  int b = 1;
  while ((1 << b) <= E) ++b;  // keys 0..E fit in b bits
  return b;
}

// Loads the ids of `steps` (<= kSteps) 32-slot steps starting at c0, all up front so the
// loads overlap; slots past n read as -1 (not local).
__device__ __forceinline__ void load_steps(const int32_t* ids, int64_t n, int64_t c0, int steps,
                                           int v[kSteps]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int64_t f = c0 + int64_t(s) * 32 + lane;
    v[s] = (s < steps && f < n) ? __ldg(ids + f) : -1;
  }
}

// hist_row[e] += number of local slots of expert e among the loaded steps (warp-cooperative).
// Non-local slots carry key E.
__device__ __forceinline__ void chunk_count(const int v[kSteps], int steps, int E, int nbits,
                                            int* hist_row) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    if (s >= steps) break;
    const int e = v[s];
    const bool loc = is_local(e, E);
    const unsigned peers = peers_of(loc ? unsigned(e) : unsigned(E), nbits);
    if (loc && lane == __ffs(peers) - 1) hist_row[e] += __popc(peers);
    __syncwarp();
  }
}

// Places every local slot of the loaded steps at run_row[e] + (rank inside the expert),
// advancing run_row[e]. Ranks follow increasing flat index.
__device__ __forceinline__ void chunk_scatter(const int v[kSteps], int steps, int64_t c0, int E,
                                              int nbits, int* run_row, int32_t* sorted_ids) {
  const int lane = threadIdx.x & 31;
  const unsigned lower = (1u << lane) - 1u;
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    if (s >= steps) break;
    const int e = v[s];
    const bool loc = is_local(e, E);
    const unsigned peers = peers_of(loc ? unsigned(e) : unsigned(E), nbits);
    if (loc) sorted_ids[run_row[e] + __popc(peers & lower)] = int32_t(c0 + int64_t(s) * 32 + lane);
    __syncwarp();
    if (loc && lane == __ffs(peers) - 1) run_row[e] += __popc(peers);
    __syncwarp();
  }
}


// Exclusive prefix sum over vals[0..count) in shared memory (count <= blockDim.x <= 1024),
// returns the total. All threads of the block must call it.
__device__ int block_exclusive_scan(int* vals, int count, int* warp_sums) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int v = tid < count ? vals[tid] : 0;
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int o = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += o;
    }
    if (lane < nwarps) warp_sums[lane] = wi - w;  // exclusive warp offsets
    if (lane == 31) warp_sums[32] = wi;           // total
  }
  __syncthreads();
  if (tid < count) vals[tid] = incl - v + warp_sums[warp];
  const int total = warp_sums[32];
  __syncthreads();
  return total;
}

// Sentinel fill and expert_ids, shared by both paths.
// cnt[e] = local slots, off[0..E] = padded offsets. Work items are distributed over
// `worker` in [0, nworkers) threads.
__device__ void fill_tail(const int* cnt, const int* off, int E, int block_m, int64_t n, int64_t cap,
                          int64_t nblocks, int32_t* sorted_ids, int32_t* expert_ids,
                          int64_t worker, int64_t nworkers) {
  const int ntp = off[E];
  // padding slots inside each expert's region
  for (int e = int(worker); e < E; e += int(nworkers)) {
    for (int i = off[e] + cnt[e]; i < off[e + 1]; ++i) sorted_ids[i] = int32_t(n);
  }
  for (int64_t i = ntp + worker; i < cap; i += nworkers) sorted_ids[i] = int32_t(n);
  const int64_t used_blocks = ntp / block_m;
  for (int64_t b = worker; b < nblocks; b += nworkers) {
    int val = -1;
    if (b < used_blocks) {
      // largest e with off[e] <= b*block_m (experts with empty regions are skipped)
      const int row = int(b * block_m);
      int lo = 0, hi = E - 1;
      while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= row) lo = mid; else hi = mid - 1;
      }
      val = lo;
    }
    expert_ids[b] = val;
  }
}

// ---- single CTA (n <= 32 chunks) ---------------------------------------------------
__global__ void __launch_bounds__(1024) align_single_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int block_m, int64_t cap, int64_t nblocks,
    int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids, int32_t* __restrict__ ntp_out,
    int32_t* __restrict__ offsets_out) {
  extern __shared__ int smem[];
  int* hist = smem;                 // [32][E]
  int* cnt = hist + 32 * E;         // [E]
  int* off = cnt + E;               // [E+1]
  int* wsum = off + E + 1;          // [33]
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < 32 * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  // warp w owns `steps` consecutive 32-slot steps, so every warp works even for small n
  const int nbits = key_bits(E);
  const int steps = int((n + 32 * 32 - 1) / (32 * 32));
  const int64_t c0 = int64_t(warp) * steps * 32;
  int v[kSteps];
  load_steps(ids, n, c0, steps, v);
  if (c0 < n) chunk_count(v, steps, E, nbits, hist + warp * E);
  __syncthreads();

  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    cnt[e] = run;
    off[e] = (run + block_m - 1) / block_m * block_m;
  }
  __syncthreads();
  const int total = block_exclusive_scan(off, E, wsum);
  if (tid == 0) off[E] = total;
  for (int i = tid; i < 32 * E; i += blockDim.x) hist[i] += off[i % E];
  __syncthreads();

  if (c0 < n) chunk_scatter(v, steps, c0, E, nbits, hist + warp * E, sorted_ids);
  fill_tail(cnt, off, E, block_m, n, cap, nblocks, sorted_ids, expert_ids, tid, blockDim.x);
  if (tid == 0) *ntp_out = off[E];
  if (offsets_out)
    for (int e = tid; e <= E; e += blockDim.x) offsets_out[e] = off[e];
}

// ---- multi CTA ---------------------------------------------------------------------
// workspace: chunk_hist [E][G] int32 | cnt [E] | off [E+1]
constexpr int kWarpsPerCta = 4;

__global__ void __launch_bounds__(32 * kWarpsPerCta) align_count_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int64_t G, int* __restrict__ chunk_hist) {
  extern __shared__ int smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* row = smem + warp * E;
  for (int i = lane; i < E; i += 32) row[i] = 0;
  __syncwarp();
  const int64_t chunk = int64_t(blockIdx.x) * kWarpsPerCta + warp;
  if (chunk >= G) return;
  int v[kSteps];
  load_steps(ids, n, chunk * kChunk, kSteps, v);
  chunk_count(v, kSteps, E, key_bits(E), row);
  for (int e = lane; e < E; e += 32) chunk_hist[int64_t(e) * G + chunk] = row[e];
}

__global__ void __launch_bounds__(1024) align_scan_kernel(int E, int block_m, int64_t G,
                                                          int* __restrict__ chunk_hist,
                                                          int* __restrict__ cnt_g,
                                                          int* __restrict__ off_g,
                                                          int32_t* __restrict__ ntp_out,
                                                          int32_t* __restrict__ offsets_out) {
  __shared__ int off[kMaxE + 1];
  __shared__ int wsum[33];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    int* h = chunk_hist + int64_t(e) * G;
    for (int64_t g = 0; g < G; ++g) {
      int c = h[g];
      h[g] = run;
      run += c;
    }
    cnt_g[e] = run;
    off[e] = (run + block_m - 1) / block_m * block_m;
  }
  __syncthreads();
  const int total = block_exclusive_scan(off, E, wsum);
  for (int e = tid; e < E; e += blockDim.x) off_g[e] = off[e];
  if (tid == 0) {
    off_g[E] = total;
    *ntp_out = total;
  }
  if (offsets_out) {
    for (int e = tid; e < E; e += blockDim.x) offsets_out[e] = off[e];
    if (tid == 0) offsets_out[E] = total;
  }
}

__global__ void __launch_bounds__(32 * kWarpsPerCta) align_scatter_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int block_m, int64_t G, int64_t cap,
    int64_t nblocks, const int* __restrict__ chunk_hist, const int* __restrict__ cnt_g,
    const int* __restrict__ off_g, int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids) {
  extern __shared__ int smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* row = smem + warp * E;
  const int64_t chunk = int64_t(blockIdx.x) * kWarpsPerCta + warp;
  if (chunk < G) {
    for (int e = lane; e < E; e += 32) row[e] = off_g[e] + chunk_hist[int64_t(e) * G + chunk];
    __syncwarp();
    int v[kSteps];
    load_steps(ids, n, chunk * kChunk, kSteps, v);
    chunk_scatter(v, kSteps, chunk * kChunk, E, key_bits(E), row, sorted_ids);
  }
  fill_tail(cnt_g, off_g, E, block_m, n, cap, nblocks, sorted_ids, expert_ids,
            int64_t(blockIdx.x) * blockDim.x + threadIdx.x, int64_t(gridDim.x) * blockDim.x);
}

}  // namespace

size_t align_workspace_bytes(int64_t n, int E) {
  const int64_t G = (n + kChunk - 1) / kChunk;
  if (G <= kSingleMaxChunks) return 0;
  return align256(uint64_t(E) * G * 4) + align256(uint64_t(E) * 4) + align256(uint64_t(E + 1) * 4);
}

cudaError_t launch_align(const int32_t* ids, int64_t n, int E, int block_m, int64_t cap,
                         int64_t nblocks, int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntp,
                         int32_t* offsets, void* workspace, cudaStream_t stream) {
  const int64_t G = (n + kChunk - 1) / kChunk;
  if (G <= kSingleMaxChunks) {
    const size_t smem = (size_t(32) * E + E + E + 1 + 33) * sizeof(int);
    cudaError_t err = cudaFuncSetAttribute(align_single_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    align_single_kernel<<<1, 1024, smem, stream>>>(ids, n, E, block_m, cap, nblocks, sorted_ids,
                                                   expert_ids, ntp, offsets);
    count_launches(1);
    return cudaGetLastError();
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* chunk_hist = reinterpret_cast<int*>(ws);
  int* cnt = reinterpret_cast<int*>(ws + align256(uint64_t(E) * G * 4));
  int* off = reinterpret_cast<int*>(ws + align256(uint64_t(E) * G * 4) + align256(uint64_t(E) * 4));
  const int64_t ctas = (G + kWarpsPerCta - 1) / kWarpsPerCta;
  const size_t smem = size_t(kWarpsPerCta) * E * sizeof(int);
  cudaError_t err = cudaFuncSetAttribute(align_count_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(align_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
  if (err != cudaSuccess) return err;
  align_count_kernel<<<unsigned(ctas), 32 * kWarpsPerCta, smem, stream>>>(ids, n, E, G, chunk_hist);
  align_scan_kernel<<<1, 1024, 0, stream>>>(E, block_m, G, chunk_hist, cnt, off, ntp, offsets);
  align_scatter_kernel<<<unsigned(ctas), 32 * kWarpsPerCta, smem, stream>>>(
      ids, n, E, block_m, G, cap, nblocks, chunk_hist, cnt, off, sorted_ids, expert_ids);
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace chord
