// chord_internal.cuh -- shared definitions of the sm_100a W4A16 MoE kernels.
//
// Repacked weight blob (written by chord_repack_weights, read by the GEMM kernels):
//
//   [0, 256)        BlobHeader
//   tiles           E * (N/128) * (K/128) tiles of 9216 bytes, tile (e, nt, kt) at
//                   256 + ((e * N/128 + nt) * K/128 + kt) * 9216
//
// A tile covers 128 physical rows x 128 K: 8192 bytes of int4 codes followed by the
// 1024 bytes of their bf16 scales, so consecutive K tiles of one row block form one
// contiguous run that a single bulk copy brings in.
//
// Codes: 8 sub-tiles of 16 rows (rb = 0..7, 1 KiB each). Inside a sub-tile the int32
// word index is
//     h*128 + g*16 + code_slot(g, t)*4 + j      (h 0..1, g 0..7, t 0..3, j 0..3)
// and holds physical row  rb*16 + 8h + g  and K range  kt*128 + 32j + 8t + [0, 8).
// code_slot(g, t) = t ^ ((g >> 1) & 3) swizzles the four 16-byte vectors of a row so
// that both ways of reading a sub-tile half are free of shared-memory bank conflicts:
// lane (g, t) of a warp reading its vector (weight streaming: 8 lanes of a phase cover
// one contiguous 128-byte span), and lane = row with t fixed across the warp (tensor core:
// 8 consecutive rows land in 8 distinct 16-byte bank groups). Inside a word, K offset u (0..7) sits in nibble
// (u >> 1) + 4 * (u & 1), so that masking nibbles {i, i+4} after a right shift by 4i
// yields the bf16 pair (u = 2i, 2i+1) in order.
//
// Scales: 128 bytes per sub-tile, bf16 index  g*8 + h*4 + j  for physical row
// rb*16 + 8h + g, group kt*4 + j.
//
// Physical row p maps to a logical row: for the down projection p itself; for gate_up
// (N = 2I) block p/16 holds gate rows 8*(p/16) + [0, 8) followed by the matching up
// rows I + 8*(p/16) + [0, 8), so a tile carries the gate and up halves of the same
// intermediate columns for the fused SiLU*up epilogue.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/chord.h"

namespace chord {

constexpr uint32_t kBlobMagic = 0x34574843u;  // "CHW4"
constexpr uint32_t kBlobVersion = 3;
constexpr uint32_t kLayoutTile128 = 2;  // 128x128 tiles, scales interleaved after codes
constexpr int kGroup = 32;
constexpr int kTileN = 128;
constexpr int kTileK = 128;
constexpr int kTileCodeBytes = kTileN * kTileK / 2;          // 8192
constexpr int kTileScaleBytes = kTileN * (kTileK / kGroup) * 2;  // 1024
constexpr int kTileBytes = kTileCodeBytes + kTileScaleBytes;     // 9216
constexpr int kHeaderBytes = 256;

struct BlobHeader {
  uint32_t magic;
  uint32_t version;
  uint32_t layout;
  uint32_t role;
  int32_t E, N, K, group;
  uint64_t tiles_offset;
  uint64_t tile_bytes;
  uint64_t total_bytes;
  uint32_t reserved[50];
};
static_assert(sizeof(BlobHeader) == kHeaderBytes, "header size");

__host__ __device__ inline uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

__host__ __device__ inline uint64_t blob_tiles_offset() { return kHeaderBytes; }
__host__ __device__ inline uint64_t blob_num_tiles(int E, int N, int K) {
  return uint64_t(E) * (N / kTileN) * (K / kTileK);
}
__host__ __device__ inline uint64_t blob_total_bytes(int E, int N, int K) {
  return align256(kHeaderBytes + blob_num_tiles(E, N, K) * kTileBytes);
}

// Logical row of physical row p in a tile-layout matrix with N physical rows.
__host__ __device__ inline int logical_row(int role, int N, int p) {
  if (role != CHORD_ROLE_GATE_UP) return p;
  int blk = p >> 4, r = p & 15;
  return r < 8 ? (blk * 8 + r) : (N / 2 + blk * 8 + (r - 8));
}

// 16-byte vector slot (0..3) of K slice t of sub-tile row g (see the layout above).
__host__ __device__ inline int code_slot(int g, int t) { return t ^ ((g >> 1) & 3); }

// Nibble slot holding K offset u (0..7) of a repacked word.
__host__ __device__ inline int nibble_slot(int u) { return (u >> 1) + 4 * (u & 1); }

// ------------------------------------------------------------------------------------
// Stream-K scratch of the weight-streaming GEMM: each of its workers (two consumer groups
// per CTA, at most kMaxStreamCtas CTAs) may leave one FP32 partial tile (8 warps x 32
// lanes x TC/2 floats) behind, announced by one flag per warp. Flags are zero between
// launches (each is reset by the worker that consumes it), so they live in the
// workspace header, which the caller zeroes once.
constexpr int kMaxStreamCtas = 256;
constexpr int kMaxStreamWorkers = 2 * kMaxStreamCtas;
constexpr uint64_t kStreamFlagBytes = uint64_t(kMaxStreamWorkers) * 8 * 4;
__host__ __device__ inline int stream_token_chunk(int block_m) { return block_m <= 8 ? 8 : (block_m <= 16 ? 16 : 32); }
__host__ __device__ inline uint64_t stream_partial_bytes(int tc) {
  return uint64_t(kMaxStreamWorkers) * 8 * 32 * (tc / 2) * 4;
}
// Header of both workspaces (forward and grouped): the device status word at offset 0,
// the stream-K flags from offset 256. Zeroed once by the caller after allocation.
constexpr uint64_t kWorkspaceHeaderBytes = CHORD_WORKSPACE_HEADER_BYTES;
static_assert(256 + 2 * kStreamFlagBytes <= kWorkspaceHeaderBytes, "workspace header");

// Workspace of chord_moe_forward:
//   [header 64 KiB: status, stream-K flags of the gate_up and down GEMMs]
//   [a: cap x I bf16][y: cap x H fp32][xs: cap x H bf16][slot_pos: T*topk i32]
//   [stream-K partials of the gate_up and down GEMMs]
// a is the SiLU*up intermediate by sorted position (row-major [cap, I]); y the expert outputs
// before the top-k weight (by flat slot [T*topk, H] on the streaming schedule, by sorted
// position in 128-column blocks [H/128][cap][128] on the tensor-core schedule, so that a
// work item writes one contiguous block); xs the hidden rows in sorted order [cap, H],
// and slot_pos the sorted position of every local flat slot (both tensor-core schedule
// only).
struct ForwardWorkspace {
  uint64_t flags_offset, a_offset, y_offset, xs_offset, slot_pos_offset, partial_offset, partial_bytes, total;
};
__host__ __device__ inline ForwardWorkspace forward_workspace(int64_t T, int topk, int E, int H,
                                                              int I, int block_m) {
  ForwardWorkspace w;
  int64_t cap = T * topk + int64_t(E) * (block_m - 1);
  w.flags_offset = 256;  // [2][kMaxStreamWorkers][8]: gate_up, down
  w.a_offset = kWorkspaceHeaderBytes;
  w.y_offset = align256(w.a_offset + uint64_t(cap) * I * 2);
  w.xs_offset = align256(w.y_offset + uint64_t(cap) * H * 4);
  w.slot_pos_offset = align256(w.xs_offset + uint64_t(cap) * H * 2);
  w.partial_offset = align256(w.slot_pos_offset + uint64_t(T) * topk * 4);
  w.partial_bytes = stream_partial_bytes(stream_token_chunk(block_m));  // per GEMM
  w.total = align256(w.partial_offset + 2 * w.partial_bytes);
  return w;
}

// ------------------------------------------------------------------------------------
// Routing tag (num_tokens_padded[1]): the block_m the routing tensors were built for.

__host__ __device__ constexpr int32_t routing_tag(int block_m) { return CHORD_ROUTING_TAG(block_m); }

// The sorted positions a forward kernel may process: num_tokens_padded[0] clamped to
// [0, cap], or 0 when num_tokens_padded[1] is not the tag of `block_m` (then
// CHORD_DEV_BLOCK_M_MISMATCH is raised and no other routing tensor may be read: with a
// smaller block_m than the routing sort used, expert_ids would be indexed past its end).
__device__ __forceinline__ int routed_positions(const int32_t* ntp, int block_m, int64_t cap, uint32_t* status) {
  if (ntp[1] != routing_tag(block_m)) {
    atomicOr(status, CHORD_DEV_BLOCK_M_MISMATCH);
    return 0;
  }
  int n = ntp[0];
  if (n < 0) n = 0;
  if (n > cap) n = int(cap);
  return n;
}

// ------------------------------------------------------------------------------------
// Host-side argument checks shared by the entry points (api.cu). fail() records the
// detail text that chord_last_error_detail() returns and passes the status through.

chord_status_t fail(chord_status_t st, const char* fmt, ...);
chord_status_t cuda_fail(cudaError_t err, const char* what);
void clear_detail();
// T, topk, E and block_m of a routing sort: ranges and a capacity below 2^31.
chord_status_t check_align_args(int64_t T, int topk, int E, int block_m);
// The current device, which must be sm_100; *num_sms receives its SM count.
chord_status_t current_device(int* num_sms);

// ------------------------------------------------------------------------------------
// PTX helpers (sm_100a)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Any on-chip wait gives up after this long, flags CHORD_DEV_TIMEOUT and unwinds.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread (up to `hint_ns`) until the phase completes,
// instead of returning at once: waiting warps then cost no issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, for at most limit_ns. Returns false (and
// raises the CTA's abort flag and the device status) when the wait gave up, or false
// alone when another thread of the CTA had aborted.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                uint32_t* status, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      if (status) atomicOr(status, CHORD_DEV_TIMEOUT);
      return false;
    }
  }
}

// The wait every kernel of the library uses: mbar_wait_limit with kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  return mbar_wait_limit(bar, parity, abort_flag, status, kWaitLimitNs);
}

// One bulk copy global -> shared, completing `bytes` of transaction on `bar`.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 eviction-priority policy (createpolicy result).
__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gsrc, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// ------------------------------------------------------------------------------------
// int4 -> bf16 dequantisation, subtract first, then scale, each rounded in BF16.
//
// 0x4300 | q is the bf16 bit pattern of 128 + q (q < 16 fills mantissa bits 0..3), so
// subtracting 136 gives q - 8 exactly; the product with the bf16 scale is rounded once
// (round-to-nearest-even), matching bf16((q - 8) * s).

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(bits));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// word: one repacked int32 (eight codes); s2: the group scale in both halves.
// out[i] = bf16 pair for K offsets (2i, 2i+1) of the word's 8-element run.
__device__ __forceinline__ void dequant8(uint32_t word, uint32_t s2, uint32_t out[4]) {
  const uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u, k136 = 0x43084308u;
  out[0] = bf16x2_mul(bf16x2_sub(lop3_and_or(word, kMask, kMagic), k136), s2);
  out[1] = bf16x2_mul(bf16x2_sub(lop3_and_or(word >> 4, kMask, kMagic), k136), s2);
  out[2] = bf16x2_mul(bf16x2_sub(lop3_and_or(word >> 8, kMask, kMagic), k136), s2);
  out[3] = bf16x2_mul(bf16x2_sub(lop3_and_or(word >> 12, kMask, kMagic), k136), s2);
}

__device__ __forceinline__ uint32_t bf16_splat(uint16_t s) { return uint32_t(s) * 0x10001u; }

// The low (hi = 0) or high (hi = 1) bf16 of `pair` in both halves (one byte permute).
__device__ __forceinline__ uint32_t bf16_splat_half(uint32_t pair, int hi) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(pair), "r"(hi ? 0x3232u : 0x1010u));
  return d;
}

// D (f32 16x8) += A (bf16 16x16, row) * B (bf16 16x8, col). Not volatile: a pure
// function of its operands, so the compiler may interleave it with independent work.
__device__ __forceinline__ void mma_bf16_16816(float c[4], const uint32_t a[4], uint32_t b0,
                                               uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

// ------------------------------------------------------------------------------------
// Programmatic dependent launch. A kernel launched with launch_pdl may start while the
// kernel before it on the stream is still running (its CTAs take the SMs the earlier
// kernel's CTAs leave); it calls grid_dep_wait() before its first access to anything
// that kernel writes, and grid_dep_wait() returns once that kernel has completed and its
// memory is visible. grid_dep_trigger() lets this kernel's own dependent launch before
// this kernel finishes. Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... Params, typename... Args>
cudaError_t launch_pdl(bool pdl, void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ------------------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files; return cudaGetLastError()).

cudaError_t launch_wait_timeout(uint32_t* status, uint64_t* elapsed_ns, uint64_t limit_ns, cudaStream_t stream);

cudaError_t launch_align(const int32_t* ids, int64_t n, int E, int block_m, int64_t cap,
                         int64_t nblocks, int32_t* sorted_ids, int32_t* expert_ids,
                         int32_t* ntp, int32_t* offsets, void* workspace, cudaStream_t stream);
// Top-k softmax router then the routing sort (one launch when T*k is small).
cudaError_t launch_router_align(const float* logits, int64_t T, int G, int k, int32_t* topk_ids,
                                float* topk_weights, int E, int block_m, int64_t cap, int64_t nblocks,
                                int32_t* sorted_ids, int32_t* expert_ids, int32_t* ntp, int32_t* offsets,
                                void* workspace, cudaStream_t stream);
size_t align_workspace_bytes(int64_t n, int E);

cudaError_t launch_repack(const int32_t* qweight, const uint16_t* scales, int E, int N, int K,
                          int role, uint8_t* blob, cudaStream_t stream);
cudaError_t launch_dequant_blob(const uint8_t* blob, int E, int N, int K, int role,
                                uint16_t* w, cudaStream_t stream);

struct ForwardArgs {
  const uint16_t* x;
  const int32_t* topk_ids;
  const float* topk_weights;
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* ntp;
  const uint8_t* w13;
  const uint8_t* w2;
  uint16_t* out;
  uint16_t* a;     // [cap, I] bf16 intermediate by sorted position
  float* y;        // fp32 expert outputs before the top-k weight: [T*topk, H] by flat slot, or
                   // [H/128][cap][128] by sorted position (y_blocked, tensor core)
  uint16_t* xs;    // [cap, H] bf16 hidden rows in sorted order (tensor-core schedule)
  int32_t* slot_pos;  // [T*topk] sorted position of each local flat slot (tensor-core schedule)
  bool y_blocked;     // y is by sorted position in 128-column blocks
  bool out_f32;       // out receives the FP32 sums (float [T, H]) instead of their BF16 rounding
  bool pdl;           // launch the streaming GEMMs and the combine early (programmatic)
  uint32_t* status;
  uint32_t* stream_flags;   // [2][kMaxStreamWorkers][8] stream-K flags (gate_up, down)
  float* stream_partial;    // [2] x stream_partial_bytes stream-K partials (gate_up, down)
  uint64_t stream_partial_bytes;
  int64_t T;
  int H, I, E, topk, block_m;
  int64_t cap;     // sorted_ids capacity
  int num_sms;
};

// Grouped operators: workspace layout for `rows` rows of x (M, or E * max_m) and E
// experts, for any unit size bm in {8, 16, 32, 64, 128, 256}.
struct GroupedWorkspace {
  int64_t max_units, max_positions, flags_offset, ntp_offset, expert_ids_offset, block_row0_offset, sorted_ids_offset,
      partial_offset, total;
};
GroupedWorkspace grouped_workspace(int64_t rows, int E);
// The routing pass: m_indices (contiguous, 16-byte aligned) or masked_m (masked) -> units
// of bm rows, bm in {8, 16, 32, 64, 128, 256}.
cudaError_t launch_grouped_route(const int32_t* m_indices, int64_t M, const int32_t* masked_m, int E,
                                 int64_t max_m, int bm, int32_t* expert_ids, int32_t* block_row0,
                                 int32_t* sorted_ids, int32_t* ntp, uint32_t* status, cudaStream_t stream);

struct GroupedArgs {
  const uint16_t* x;        // [rows, K]
  int64_t rows;
  int K, N, E, role;
  const uint8_t* w;         // blob
  uint16_t* out;            // [rows, N]
  const int32_t* sorted_ids;
  const int32_t* expert_ids;
  const int32_t* block_row0;
  const int32_t* ntp;
  int bm;                   // positions per unit
  int64_t cap;              // sorted_ids capacity
  uint32_t* status;
  uint32_t* stream_flags;   // [kMaxStreamWorkers][8] stream-K flags
  float* stream_partial;    // stream-K partials (token chunk up to 32)
  int num_sms;
};
// The GEMM of the grouped operators: out[row] = x[row] . W[e]^T for every valid row.
cudaError_t launch_tc_grouped(const GroupedArgs& g, cudaStream_t stream);
cudaError_t launch_stream_grouped(const GroupedArgs& g, cudaStream_t stream);  // token chunk = g.bm

// Exchange steps of sharded deployments (shard.cu).
cudaError_t launch_ep_route(const int32_t* topk_ids, int64_t T, int topk, int E_rank, int W, int32_t* ids_tw,
                            int32_t* row_of, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_pack(const uint16_t* x, const int32_t* topk_ids, const float* topk_weights, int64_t T, int H,
                           int topk, int E_rank, int W, const int32_t* send_rows, const int32_t* rank_offsets,
                           uint16_t* send_x, int32_t* send_ids, float* send_w, int32_t* row_of, int num_sms,
                           cudaStream_t stream);
cudaError_t launch_ep_combine(const uint16_t* back, const int32_t* row_of, int64_t rows_cap, int64_t T, int H, int W,
                              uint16_t* out, int num_sms, cudaStream_t stream);
cudaError_t launch_round_bf16(const float* in, int64_t n, uint16_t* out, int num_sms, cudaStream_t stream);
// The ranks' FP32 partials and BF16 outputs of the tensor-parallel reduction, by pointer.
constexpr int kMaxTpRanks = 64;
struct TpPeers {
  const float* in[kMaxTpRanks];
  uint16_t* out[kMaxTpRanks];
};
cudaError_t launch_tp_reduce_round(const TpPeers& peers, int W, int rank, int64_t n, int num_sms, cudaStream_t stream);

// Adds n to the process-wide kernel launch counter (chord_launch_count).
void count_launches(int n);

// `mid` (may be null) is recorded on the stream between the gate_up and down GEMMs.
cudaError_t launch_validate(const ForwardArgs& a, cudaStream_t stream);
// Records a caller's timing event on `stream`. Under stream capture the record becomes an
// event node of the graph (a plain record would only order the capture), so a captured
// forward still times its kernels when the graph is replayed.
inline cudaError_t record_timing_event(cudaEvent_t ev, cudaStream_t stream) {
  return cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
}

// `first` (if set) is recorded right before the gate_up GEMM kernel, `mid` between the two
// GEMM kernels.
cudaError_t launch_stream_gemms(const ForwardArgs& a, cudaStream_t stream, cudaEvent_t first, cudaEvent_t mid);
cudaError_t launch_tc_gemms(const ForwardArgs& a, cudaStream_t stream, cudaEvent_t first, cudaEvent_t mid);
// xs <- the hidden rows in routing order [cap, H] (tensor-core schedule).
cudaError_t launch_permute_rows(const ForwardArgs& a, cudaStream_t stream);
cudaError_t launch_combine(const ForwardArgs& a, cudaStream_t stream);

}  // namespace chord
