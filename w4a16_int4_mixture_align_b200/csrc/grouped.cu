// grouped.cu -- routing pass of the grouped operators ("Gruppierte SM90-Kernel").
//
// The grouped layouts keep each expert's rows consecutive in x: the contiguous layout
// concatenates them in runs padded to 128 rows and labels rows with m_indices (-1 for
// padding); the masked layout gives every expert a fixed budget of max_m rows of which
// masked_m[e] are valid. The GEMM kernels of this library consume the indexed routing
// form (units of bm positions, one expert per unit), so one pass turns either layout
// into that form without touching x:
//   expert_ids[u]  the expert of unit u (units without a valid row are not emitted),
//   block_row0[u]  the x row of the unit's first position (a unit's rows are
//                  consecutive in x, so the tensor-core schedule loads them as one box),
//   sorted_ids[p]  the x row of position p, or -1 where the row belongs to no expert,
//   ntp            number of units * bm.
// bm is the schedule's unit: 8, 16 or 32 rows for the weight-streaming GEMM (one token
// chunk per unit, so no empty chunk is ever visited), 32 to 256 for the tensor cores.
// With bm = 256 two neighbouring 128-row blocks of the same expert form one unit (twice
// the reuse of every dequantised weight tile); a block whose neighbour belongs to another
// expert is a unit of its own with an empty second half.
//
// One CTA does the pass. Masked: a thread per expert counts its units, one block-wide
// prefix sum numbers them, a warp per expert writes them. Contiguous: batches of 256
// chunks (a chunk = bm/128 blocks of 128 rows when bm = 256, else one block); a warp
// reads four chunks at a time with 16-byte loads and keeps each block's valid rows as a
// 128-bit map in shared memory, a prefix sum over the chunks' unit counts numbers the
// units, and each lane then writes the routing entries of four rows with one 16-byte store.
#include <climits>

#include "chord_internal.cuh"

namespace chord {
namespace {

constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kBatch = 256;                    // contiguous chunks per pass
constexpr int kPerWarp = kBatch / kRouteWarps;  // chunks a warp classifies per batch

__device__ __forceinline__ int warp_min(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_max(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Exclusive prefix sum of v over the threads of a 1024-thread block; every thread must
// call it. Returns the sum over the threads before this one and writes the block total
// to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = s_warp[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    s_warp[lane] = wi - w;
    if (lane == 31) s_warp[32] = wi;
  }
  __syncthreads();
  const int r = s_warp[warp] + incl - v;
  *total = s_warp[32];
  __syncthreads();  // s_warp may be reused right after
  return r;
}

// four m_indices entries from row `row` (16-byte aligned when row + 3 < M); rows past M
// read as padding
__device__ __forceinline__ int4 load_ids4(const int32_t* __restrict__ m, int64_t row, int64_t M) {
  if (row + 3 < M) return __ldg(reinterpret_cast<const int4*>(m + row));
  int4 v = make_int4(-1, -1, -1, -1);
  if (row < M) v.x = __ldg(m + row);
  if (row + 1 < M) v.y = __ldg(m + row + 1);
  if (row + 2 < M) v.z = __ldg(m + row + 2);
  return v;
}

__device__ __forceinline__ void st_int4(int32_t* p, int a, int b, int c, int d) {
  *reinterpret_cast<int4*>(p) = make_int4(a, b, c, d);
}

__global__ void __launch_bounds__(kRouteThreads) grouped_route_masked_kernel(
    const int32_t* __restrict__ masked_m, int E, int64_t max_m, int bm, int32_t* __restrict__ expert_ids,
    int32_t* __restrict__ block_row0, int32_t* __restrict__ sorted_ids, int32_t* __restrict__ ntp,
    uint32_t* __restrict__ status) {
  __shared__ int s_warp[33];
  __shared__ int s_base[kRouteThreads];
  __shared__ int s_rows[kRouteThreads];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bool bad = false;
  int cnt = 0, units = 0;
  if (tid < E) {
    int64_t v = __ldg(masked_m + tid);
    if (v < 0 || v > max_m) {
      bad = true;
      v = v < 0 ? 0 : max_m;
    }
    cnt = int(v);
    units = (cnt + bm - 1) / bm;
  }
  int total = 0;
  const int base = block_exclusive_scan(units, s_warp, &total);
  s_base[tid] = base;
  s_rows[tid] = cnt;
  __syncthreads();
  const int qpu = bm / 4;  // 16-byte vectors per unit
  for (int e = warp; e < E; e += kRouteWarps) {
    const int rows = s_rows[e], u0 = s_base[e];
    const int nvec = ((rows + bm - 1) / bm) * qpu;
    const int64_t erow = int64_t(e) * max_m;
    for (int v = lane; v < nvec; v += 32) {
      const int j = v / qpu, r = (v - j * qpu) * 4 + j * bm;  // row within the expert
      const int u = u0 + j;
      if (r == j * bm) {
        expert_ids[u] = e;
        block_row0[u] = int32_t(erow + int64_t(j) * bm);
      }
      const int32_t f = int32_t(erow + r);
      st_int4(sorted_ids + int64_t(u) * bm + (r - j * bm), r < rows ? f : -1, r + 1 < rows ? f + 1 : -1,
              r + 2 < rows ? f + 2 : -1, r + 3 < rows ? f + 3 : -1);
    }
  }
  if (tid == 0) {
    ntp[0] = total * bm;
    ntp[1] = routing_tag(bm);
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(status, CHORD_DEV_ROUTING_INVALID);
}

// Contiguous layout. U = 2 when bm = 256 (chunk = two blocks), else 1; sub-blocks of
// sb = min(bm, 128) rows are the units of a block when bm <= 128.
__global__ void __launch_bounds__(kRouteThreads) grouped_route_contiguous_kernel(
    const int32_t* __restrict__ m_indices, int64_t M, int E, int bm, int64_t n_chunks,
    int32_t* __restrict__ expert_ids, int32_t* __restrict__ block_row0, int32_t* __restrict__ sorted_ids,
    int32_t* __restrict__ ntp, uint32_t* __restrict__ status) {
  __shared__ uint32_t s_bits[kBatch][2][4];  // valid rows of each block, bit r%32 of word r/32
  __shared__ int s_e[kBatch][2];             // expert of each block, -1 when it is skipped
  __shared__ int s_base[kBatch];             // first unit of each chunk
  __shared__ int s_warp[33];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int U = bm == 256 ? 2 : 1;
  const int sb = bm < 128 ? bm : 128;  // rows per unit inside one block
  const int nsub = 128 / sb;
  int done = 0;  // units of earlier batches
  bool bad = false;

  for (int64_t c0 = 0; c0 < n_chunks; c0 += kBatch) {
    // ---- classify: warp w takes chunks w*kPerWarp .. +kPerWarp-1 of the batch, loading
    // kLoadAhead chunks before reducing any (registers allow no more at 1024 threads)
    constexpr int kLoadAhead = 4;
#pragma unroll 1
    for (int j0 = 0; j0 < kPerWarp; j0 += kLoadAhead) {
      int4 v[kLoadAhead][2];
#pragma unroll
      for (int j = 0; j < kLoadAhead; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t c = c0 + warp * kPerWarp + j0 + j;
          v[j][h] = make_int4(-1, -1, -1, -1);
          if (h < U && c < n_chunks) v[j][h] = load_ids4(m_indices, (c * U + h) * 128 + 4 * lane, M);
        }
#pragma unroll
      for (int j = 0; j < kLoadAhead; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int4 q = v[j][h];
          const int ids[4] = {q.x, q.y, q.z, q.w};
          int lo = INT_MAX, hi = -1;
          uint32_t nib = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b)
            if (ids[b] >= 0) {
              lo = min(lo, ids[b]);
              hi = max(hi, ids[b]);
              nib |= 1u << b;
            }
          lo = warp_min(lo);
          hi = warp_max(hi);
          int e = -1;
          if (hi >= 0) {
            if (lo != hi || hi >= E) bad = true;  // mixed block or unknown expert: skipped
            else e = hi;
          }
          if (e < 0) nib = 0;
          uint32_t word[4];
#pragma unroll
          for (int w = 0; w < 4; ++w)
            word[w] = __reduce_or_sync(0xffffffffu, (lane >> 3) == w ? nib << (4 * (lane & 7)) : 0u);
          if (lane == 0) {
            const int i = warp * kPerWarp + j0 + j;
#pragma unroll
            for (int w = 0; w < 4; ++w) s_bits[i][h][w] = word[w];
            s_e[i][h] = e;
          }
        }
    }
    __syncthreads();
    // ---- units per chunk, numbered by a prefix sum
    int cnt = 0;
    if (tid < kBatch) {
      const int e0 = s_e[tid][0], e1 = s_e[tid][1];
      if (U == 2) {
        cnt = (e0 >= 0 && e0 == e1) ? 1 : int(e0 >= 0) + int(e1 >= 0);
      } else if (e0 >= 0) {
        for (int s = 0; s < nsub; ++s) {
          // sub-block s: bits [s*sb, (s+1)*sb) of the block's map
          const int b0 = s * sb;
          uint32_t any = 0;
          for (int w = b0 >> 5; w <= (b0 + sb - 1) >> 5; ++w) {
            uint32_t m = s_bits[tid][0][w];
            if (sb < 32) m = (m >> (b0 & 31)) & ((1u << sb) - 1u);
            any |= m;
          }
          cnt += any != 0;
        }
      }
    }
    int total = 0;
    const int base = block_exclusive_scan(cnt, s_warp, &total);
    if (tid < kBatch) s_base[tid] = done + base;
    __syncthreads();
    // ---- write: a warp per chunk, each lane four rows of a block with one 16-byte store
    for (int i = warp; i < kBatch; i += kRouteWarps) {
      const int64_t c = c0 + i;
      if (c >= n_chunks) break;
      const int e0 = s_e[i][0], e1 = s_e[i][1];
      const bool merged = U == 2 && e0 >= 0 && e0 == e1;
      for (int h = 0; h < U; ++h) {
        const int e = h == 0 ? e0 : e1;
        if (e < 0) continue;
        const int r = 4 * lane;  // rows r .. r+3 of this block
        const int64_t brow = (c * U + h) * 128;
        const uint32_t bits = (s_bits[i][h][r >> 5] >> (r & 31)) & 0xFu;
        int u, off;
        bool head;
        if (U == 2) {
          u = s_base[i] + ((h == 1 && !merged && e0 >= 0) ? 1 : 0);
          off = merged ? 128 * h + r : r;
          head = lane == 0 && !(merged && h == 1);
        } else {
          // sub-block s of this lane's rows; units are the non-empty sub-blocks in order
          const int s = r / sb;
          uint32_t nonempty_before = 0;
          bool mine = false;
          for (int t = 0; t <= s; ++t) {
            const int b0 = t * sb;
            uint32_t any = 0;
            for (int w = b0 >> 5; w <= (b0 + sb - 1) >> 5; ++w) {
              uint32_t m = s_bits[i][0][w];
              if (sb < 32) m = (m >> (b0 & 31)) & ((1u << sb) - 1u);
              any |= m;
            }
            if (t < s) nonempty_before += any != 0;
            else mine = any != 0;
          }
          if (!mine) continue;
          u = s_base[i] + int(nonempty_before);
          off = r - s * sb;
          head = off == 0;
        }
        if (head) {
          expert_ids[u] = e;
          block_row0[u] = int32_t(brow + (U == 2 ? 0 : r));
        }
        const int32_t f = int32_t(brow + r);
        st_int4(sorted_ids + int64_t(u) * bm + off, (bits & 1u) ? f : -1, (bits & 2u) ? f + 1 : -1,
                (bits & 4u) ? f + 2 : -1, (bits & 8u) ? f + 3 : -1);
        if (U == 2 && !merged) st_int4(sorted_ids + int64_t(u) * bm + 128 + r, -1, -1, -1, -1);
      }
    }
    done += total;
    __syncthreads();  // the shared arrays are rewritten by the next batch
  }
  if (tid == 0) {
    ntp[0] = done * bm;
    ntp[1] = routing_tag(bm);
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(status, CHORD_DEV_ROUTING_INVALID);
}

}  // namespace

GroupedWorkspace grouped_workspace(int64_t rows, int E) {
  GroupedWorkspace w;
  // units: at most one per 8 rows plus one partial unit per expert; positions: at most
  // 256 per 128-row block plus 256 per expert
  w.max_units = (rows + 7) / 8 + E;
  w.max_positions = ((rows + 127) / 128 + E) * 256;
  auto up = [](int64_t b) { return (b + 255) / 256 * 256; };
  w.flags_offset = 256;  // stream-K flags, inside the zero-once header
  w.ntp_offset = int64_t(kWorkspaceHeaderBytes);
  w.expert_ids_offset = w.ntp_offset + 256;
  w.block_row0_offset = w.expert_ids_offset + up(w.max_units * 4);
  w.sorted_ids_offset = w.block_row0_offset + up(w.max_units * 4);
  w.partial_offset = w.sorted_ids_offset + up(w.max_positions * 4);
  w.total = w.partial_offset + int64_t(stream_partial_bytes(32));
  return w;
}

cudaError_t launch_grouped_route(const int32_t* m_indices, int64_t M, const int32_t* masked_m, int E,
                                 int64_t max_m, int bm, int32_t* expert_ids, int32_t* block_row0,
                                 int32_t* sorted_ids, int32_t* ntp, uint32_t* status, cudaStream_t stream) {
  if (masked_m) {
    grouped_route_masked_kernel<<<1, kRouteThreads, 0, stream>>>(masked_m, E, max_m, bm, expert_ids, block_row0,
                                                                 sorted_ids, ntp, status);
  } else {
    const int U = bm == 256 ? 2 : 1;
    const int64_t n_chunks = ((M + 127) / 128 + U - 1) / U;
    grouped_route_contiguous_kernel<<<1, kRouteThreads, 0, stream>>>(m_indices, M, E, bm, n_chunks, expert_ids,
                                                                     block_row0, sorted_ids, ntp, status);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace chord
