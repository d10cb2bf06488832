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
//                    scatter + fill kernel, histograms in the caller's workspace. A chunk
//                    (one warp's run) is 256 slots, so a prefill batch spreads over
//                    hundreds of warps, unless E x chunks would pass 2^17 histogram
//                    entries; then it is 1024 slots (the workspace stays within what the
//                    no-allocation variant's static scratch holds).
#include <math.h>

#include "chord_internal.cuh"

namespace chord {
namespace {

constexpr int kChunk = 1024;       // flat slots per warp chunk (largest)
constexpr int kSteps = kChunk / 32;
constexpr int kChunkSmall = 256;   // multi-CTA path, when the histograms stay small
constexpr int64_t kMaxHistEntries = int64_t(1) << 17;

// Slots per warp chunk of the multi-CTA path for n slots and E experts.
__host__ __device__ inline int multi_chunk(int64_t n, int E) {
  const int64_t g = (n + kChunkSmall - 1) / kChunkSmall;
  return int64_t(E) * g <= kMaxHistEntries ? kChunkSmall : kChunk;
}
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

// ---- single CTA (n <= kSingleMaxChunks chunks) ---------------------------------------
// The whole sort by one CTA of 1024 threads; `smem` holds (32 + 2) * E + 34 ints.
__device__ __forceinline__ void align_single_body(
    const int32_t* __restrict__ ids, int64_t n, int E, int block_m, int64_t cap, int64_t nblocks,
    int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids, int32_t* __restrict__ ntp_out,
    int32_t* __restrict__ offsets_out, int* smem) {
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
  if (tid == 0) {
    ntp_out[0] = off[E];
    ntp_out[1] = routing_tag(block_m);
  }
  if (offsets_out)
    for (int e = tid; e <= E; e += blockDim.x) offsets_out[e] = off[e];
}

__global__ void __launch_bounds__(1024) align_single_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int block_m, int64_t cap, int64_t nblocks,
    int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids, int32_t* __restrict__ ntp_out,
    int32_t* __restrict__ offsets_out) {
  extern __shared__ int smem[];
  align_single_body(ids, n, E, block_m, cap, nblocks, sorted_ids, expert_ids, ntp_out, offsets_out, smem);
}

// ---- router: top-k softmax routing, one warp per token ------------------------------
// Lane l holds the logits of experts l, l + 32, ... (PER slots). Each lane keeps its
// best unselected slot; every round the warp takes the largest of them (larger value,
// or the lower id on equal values), and only the lane that supplied it rescans. Lane
// r % 32 ends with the expert of rank r (descending logit, ties to the lower id).
constexpr int kNoExpert = 0x7fffffff;

template <int PER>
__device__ __forceinline__ void router_token(const float* __restrict__ row, int G, int k, int lane,
                                             int32_t* __restrict__ ids_out, float* __restrict__ w_out) {
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < G ? __ldg(row + e) : -INFINITY;
  }
  uint32_t taken = 0;
  // this lane's best unselected slot (ascending e: strictly greater keeps the lower id)
  auto local_best = [&](float& bv, int& bi) {
    bv = -INFINITY;
    bi = kNoExpert;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      if (e < G && !((taken >> i) & 1u) && (bi == kNoExpert || v[i] > bv)) {
        bv = v[i];
        bi = e;
      }
    }
  };
  float lv;
  int li;
  local_best(lv, li);
  int id_a = 0, id_b = 0;  // ranks lane and 32 + lane
  float l_a = -INFINITY, l_b = -INFINITY;
  for (int r = 0; r < k; ++r) {
    float bv = lv;
    int bi = li;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != kNoExpert && (bi == kNoExpert || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if (r == lane) {
      id_a = bi;
      l_a = bv;
    } else if (r == lane + 32) {
      id_b = bi;
      l_b = bv;
    }
    if (li == bi) {  // this lane supplied the winner: mark it and find its next best
      taken |= 1u << (bi >> 5);
      local_best(lv, li);
    }
  }
  // weights: softmax over the chosen logits, relative to the largest (rank 0)
  const float l0 = __shfl_sync(0xffffffffu, l_a, 0);
  const float e_a = lane < k ? expf(l_a - l0) : 0.f;
  const float e_b = lane + 32 < k ? expf(l_b - l0) : 0.f;
  float part = e_a + e_b;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane < k) {
    ids_out[lane] = id_a;
    w_out[lane] = e_a / part;
  }
  if (lane + 32 < k) {
    ids_out[lane + 32] = id_b;
    w_out[lane + 32] = e_b / part;
  }
}

template <int PER>
__device__ __forceinline__ void route_tokens(const float* __restrict__ logits, int64_t T, int G, int k,
                                             int32_t* __restrict__ topk_ids, float* __restrict__ topk_weights,
                                             int64_t warp0, int64_t nwarps, int lane) {
  for (int64_t t = warp0; t < T; t += nwarps)
    router_token<PER>(logits + t * G, G, k, lane, topk_ids + t * k, topk_weights + t * k);
}

// Slots per lane: the smallest instantiated count that covers G.
__device__ __forceinline__ void route_tokens_any(const float* __restrict__ logits, int64_t T, int G, int k,
                                                 int32_t* __restrict__ topk_ids, float* __restrict__ topk_weights,
                                                 int64_t warp0, int64_t nwarps, int lane) {
  const int per = (G + 31) / 32;
  if (per <= 4) route_tokens<4>(logits, T, G, k, topk_ids, topk_weights, warp0, nwarps, lane);
  else if (per <= 8) route_tokens<8>(logits, T, G, k, topk_ids, topk_weights, warp0, nwarps, lane);
  else if (per <= 12) route_tokens<12>(logits, T, G, k, topk_ids, topk_weights, warp0, nwarps, lane);
  else if (per <= 16) route_tokens<16>(logits, T, G, k, topk_ids, topk_weights, warp0, nwarps, lane);
  else route_tokens<32>(logits, T, G, k, topk_ids, topk_weights, warp0, nwarps, lane);
}

__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits, int64_t T, int G,
                                                          int k, int32_t* __restrict__ topk_ids,
                                                          float* __restrict__ topk_weights) {
  route_tokens_any(logits, T, G, k, topk_ids, topk_weights,
                   int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5),
                   int64_t(gridDim.x) * (blockDim.x >> 5), threadIdx.x & 31);
}

// Router and sort fused in one CTA, for batches of at most 8 tokens: the warps route the
// tokens, then the CTA sorts the ids it has just written (visible after the barrier).
// Larger batches route on many CTAs first: measured, one SM routing 32 tokens took 4 us
// more than a routing kernel plus the sort, while up to 8 tokens the saved launch wins.
constexpr int kFusedMaxTokens = 8;

__global__ void __launch_bounds__(1024) router_align_single_kernel(
    const float* __restrict__ logits, int64_t T, int G, int k, int32_t* __restrict__ topk_ids,
    float* __restrict__ topk_weights, int E, int block_m, int64_t cap, int64_t nblocks,
    int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids, int32_t* __restrict__ ntp_out,
    int32_t* __restrict__ offsets_out) {
  extern __shared__ int smem[];
  route_tokens_any(logits, T, G, k, topk_ids, topk_weights, threadIdx.x >> 5, blockDim.x >> 5, threadIdx.x & 31);
  __syncthreads();
  align_single_body(topk_ids, T * k, E, block_m, cap, nblocks, sorted_ids, expert_ids, ntp_out, offsets_out,
                    smem);
}


// ---- multi CTA ---------------------------------------------------------------------
// workspace: chunk_hist [E][G] int32 | cnt [E]
constexpr int kWarpsPerCta = 4;

__global__ void __launch_bounds__(32 * kWarpsPerCta) align_count_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int64_t G, int csz, int* __restrict__ chunk_hist) {
  extern __shared__ int smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* row = smem + warp * E;
  for (int i = lane; i < E; i += 32) row[i] = 0;
  __syncwarp();
  const int64_t chunk = int64_t(blockIdx.x) * kWarpsPerCta + warp;
  if (chunk >= G) return;
  int v[kSteps];
  load_steps(ids, n, chunk * csz, csz / 32, v);
  chunk_count(v, csz / 32, E, key_bits(E), row);
  for (int e = lane; e < E; e += 32) chunk_hist[int64_t(e) * G + chunk] = row[e];
}

// A warp per expert (32 experts per CTA): the exclusive prefix of the expert's run counts,
// in place, over windows of 32 x R runs (each lane loads its R consecutive counts at
// once: one round trip per window), and the expert's total. The experts' offsets are
// scanned by every scatter CTA itself, so no single CTA walks all experts.
__global__ void __launch_bounds__(1024) align_scan_kernel(int E, int64_t G, int* __restrict__ chunk_hist,
                                                          int* __restrict__ cnt_g) {
  const int lane = threadIdx.x & 31;
  const int e = int(blockIdx.x) * 32 + (threadIdx.x >> 5);
  if (e >= E) return;
  constexpr int R = 8;
  int* h = chunk_hist + int64_t(e) * G;
  int run = 0;
  for (int64_t base = 0; base < G; base += 32 * R) {
    int c[R];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int64_t g = base + lane * R + i;
      c[i] = g < G ? h[g] : 0;
    }
    int lsum = 0;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int x = c[i];
      c[i] = lsum;
      lsum += x;
    }
    int incl = lsum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    const int excl = run + incl - lsum;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int64_t g = base + lane * R + i;
      if (g < G) h[g] = excl + c[i];
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) cnt_g[e] = run;
}

// Exclusive prefix of vals[0, count) in place for any count (each thread sums a run of
// consecutive values, the runs' sums are scanned across the block); returns the total.
// tmp holds blockDim.x ints, warp_sums 33.
__device__ int block_exclusive_scan_runs(int* vals, int count, int* tmp, int* warp_sums) {
  const int tid = threadIdx.x;
  const int per = (count + int(blockDim.x) - 1) / int(blockDim.x);
  const int b = tid * per;
  int sum = 0;
  for (int i = 0; i < per; ++i)
    if (b + i < count) sum += vals[b + i];
  tmp[tid] = sum;
  __syncthreads();
  const int total = block_exclusive_scan(tmp, int(blockDim.x), warp_sums);
  int run = tmp[tid];
  for (int i = 0; i < per; ++i)
    if (b + i < count) {
      const int x = vals[b + i];
      vals[b + i] = run;
      run += x;
    }
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(32 * kWarpsPerCta) align_scatter_kernel(
    const int32_t* __restrict__ ids, int64_t n, int E, int block_m, int64_t G, int64_t cap,
    int64_t nblocks, int csz, const int* __restrict__ chunk_hist, const int* __restrict__ cnt_g,
    int32_t* __restrict__ sorted_ids, int32_t* __restrict__ expert_ids, int32_t* __restrict__ ntp_out,
    int32_t* __restrict__ offsets_out) {
  extern __shared__ int smem[];
  __shared__ int wsum[33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* row = smem + warp * E;
  // the experts' padded offsets, scanned by this CTA: off[e] (E + 1 entries)
  int* off = smem + kWarpsPerCta * E;
  int* tmp = off + E + 1;
  for (int e = threadIdx.x; e < E; e += blockDim.x) off[e] = (cnt_g[e] + block_m - 1) / block_m * block_m;
  __syncthreads();
  const int total = block_exclusive_scan_runs(off, E, tmp, wsum);
  if (threadIdx.x == 0) off[E] = total;
  __syncthreads();
  if (blockIdx.x == 0) {
    if (threadIdx.x == 0) {
      ntp_out[0] = total;
      ntp_out[1] = routing_tag(block_m);
    }
    if (offsets_out)
      for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets_out[e] = off[e];
  }
  const int64_t chunk = int64_t(blockIdx.x) * kWarpsPerCta + warp;
  if (chunk < G) {
    for (int e = lane; e < E; e += 32) row[e] = off[e] + chunk_hist[int64_t(e) * G + chunk];
    __syncwarp();
    int v[kSteps];
    load_steps(ids, n, chunk * csz, csz / 32, v);
    chunk_scatter(v, csz / 32, chunk * csz, E, key_bits(E), row, sorted_ids);
  }
  fill_tail(cnt_g, off, E, block_m, n, cap, nblocks, sorted_ids, expert_ids,
            int64_t(blockIdx.x) * blockDim.x + threadIdx.x, int64_t(gridDim.x) * blockDim.x);
}

}  // namespace

size_t align_workspace_bytes(int64_t n, int E) {
  if ((n + kChunk - 1) / kChunk <= kSingleMaxChunks) return 0;
  const int csz = multi_chunk(n, E);
  const int64_t G = (n + csz - 1) / csz;
  return align256(uint64_t(E) * G * 4) + align256(uint64_t(E) * 4);
}

cudaError_t launch_align(const int32_t* ids, int64_t n, int E, int block_m, int64_t cap,
                         int64_t nblocks, int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntp,
                         int32_t* offsets, void* workspace, cudaStream_t stream) {
  if ((n + kChunk - 1) / kChunk <= kSingleMaxChunks) {
    const size_t smem = (size_t(32) * E + E + E + 1 + 33) * sizeof(int);
    cudaError_t err = cudaFuncSetAttribute(align_single_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    align_single_kernel<<<1, 1024, smem, stream>>>(ids, n, E, block_m, cap, nblocks, sorted_ids,
                                                   expert_ids, ntp, offsets);
    count_launches(1);
    return cudaGetLastError();
  }
  const int csz = multi_chunk(n, E);
  const int64_t G = (n + csz - 1) / csz;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* chunk_hist = reinterpret_cast<int*>(ws);
  int* cnt = reinterpret_cast<int*>(ws + align256(uint64_t(E) * G * 4));
  const int64_t ctas = (G + kWarpsPerCta - 1) / kWarpsPerCta;
  const size_t smem = size_t(kWarpsPerCta) * E * sizeof(int);
  // scatter: the warps' rows, then the experts' offsets (E + 1) and the scan's run sums
  const size_t smem_scatter = smem + (size_t(E) + 1 + 32 * kWarpsPerCta) * sizeof(int);
  cudaError_t err = cudaFuncSetAttribute(align_count_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(align_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem_scatter));
  if (err != cudaSuccess) return err;
  align_count_kernel<<<unsigned(ctas), 32 * kWarpsPerCta, smem, stream>>>(ids, n, E, G, csz, chunk_hist);
  align_scan_kernel<<<unsigned((E + 31) / 32), 1024, 0, stream>>>(E, G, chunk_hist, cnt);
  align_scatter_kernel<<<unsigned(ctas), 32 * kWarpsPerCta, smem_scatter, stream>>>(
      ids, n, E, block_m, G, cap, nblocks, csz, chunk_hist, cnt, sorted_ids, expert_ids, ntp, offsets);
  count_launches(3);
  return cudaGetLastError();
}

cudaError_t launch_router_align(const float* logits, int64_t T, int G, int k, int32_t* topk_ids,
                                float* topk_weights, int E, int block_m, int64_t cap, int64_t nblocks,
                                int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntp, int32_t* offsets,
                                void* workspace, cudaStream_t stream) {
  const int64_t n = T * k;
  const int64_t G_chunks = (n + kChunk - 1) / kChunk;
  if (T <= kFusedMaxTokens && G_chunks <= kSingleMaxChunks) {
    const size_t smem = (size_t(32) * E + E + E + 1 + 33) * sizeof(int);
    cudaError_t err = cudaFuncSetAttribute(router_align_single_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    router_align_single_kernel<<<1, 1024, smem, stream>>>(logits, T, G, k, topk_ids, topk_weights, E, block_m, cap,
                                                          nblocks, sorted_ids, expert_ids, ntp, offsets);
    count_launches(1);
    return cudaGetLastError();
  }
  int64_t ctas = (T + 7) / 8;
  const int64_t max_ctas = 148 * 8;
  if (ctas > max_ctas) ctas = max_ctas;
  router_topk_kernel<<<unsigned(ctas), 256, 0, stream>>>(logits, T, G, k, topk_ids, topk_weights);
  count_launches(1);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_align(topk_ids, n, E, block_m, cap, nblocks, sorted_ids, expert_ids, ntp, offsets, workspace,
                      stream);
}

}  // namespace chord
