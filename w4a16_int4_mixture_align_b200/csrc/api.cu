// api.cu -- the C ABI declared in include/chord.h: argument checks, the prepared-weight
// registry, the memoised schedule selector and the launch sequence of the layer.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>
#include <unordered_map>

#include "chord_internal.cuh"

namespace chord {
namespace {

thread_local char g_detail[512] = "";
thread_local cudaEvent_t g_timing[4] = {nullptr, nullptr, nullptr, nullptr};
thread_local bool g_timing_on = false;
std::atomic<uint64_t> g_launches{0};

struct DeviceInfo {
  bool ok = false;
  int num_sms = 0;
  int major = 0, minor = 0;
};

std::mutex g_mu;
std::unordered_map<int, DeviceInfo> g_devices;

struct BlobInfo {
  int E, N, K, role;
  size_t bytes;
};
std::unordered_map<const void*, BlobInfo> g_blobs;
std::map<std::tuple<int64_t, int, int, int, int, int>, int> g_select_cache;

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

}  // namespace

chord_status_t fail(chord_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
  return st;
}

chord_status_t cuda_fail(cudaError_t err, const char* what) {
  return fail(CHORD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

void clear_detail() { g_detail[0] = 0; }

chord_status_t current_device(int* num_sms) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  DeviceInfo d;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_devices.find(dev);
    if (it == g_devices.end()) {
      DeviceInfo nd;
      cudaDeviceGetAttribute(&nd.major, cudaDevAttrComputeCapabilityMajor, dev);
      cudaDeviceGetAttribute(&nd.minor, cudaDevAttrComputeCapabilityMinor, dev);
      cudaDeviceGetAttribute(&nd.num_sms, cudaDevAttrMultiProcessorCount, dev);
      nd.ok = (nd.major == 10 && nd.minor == 0);
      it = g_devices.emplace(dev, nd).first;
    }
    d = it->second;
  }
  if (num_sms) *num_sms = d.num_sms;
  if (!d.ok)
    return fail(CHORD_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, d.major,
                d.minor);
  return CHORD_OK;
}

chord_status_t check_align_args(int64_t T, int topk, int E, int block_m) {
  if (T < 0 || topk < 1 || topk > 64)
    return fail(CHORD_ERR_INVALID_ARG, "T=%lld topk=%d", (long long)T, topk);
  if (E < 1 || E > 1024) return fail(CHORD_ERR_UNSUPPORTED, "E=%d outside [1, 1024]", E);
  if (block_m < 1 || block_m > 256)
    return fail(CHORD_ERR_UNSUPPORTED, "block_m=%d outside [1, 256]", block_m);
  // bounded before multiplying, so the product below cannot overflow
  const int64_t lim = int64_t(1) << 31;
  if (T >= lim / topk) return fail(CHORD_ERR_UNSUPPORTED, "T*topk (T=%lld, topk=%d) >= 2^31", (long long)T, topk);
  const int64_t cap = T * topk + int64_t(E) * (block_m - 1);
  if (cap >= lim) return fail(CHORD_ERR_UNSUPPORTED, "routing capacity %lld >= 2^31", (long long)cap);
  return CHORD_OK;
}

void count_launches(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }

}  // namespace chord

using namespace chord;

extern "C" {

const char* chord_status_string(int status) {
  switch (status) {
    case CHORD_OK: return "CHORD_OK";
    case CHORD_ERR_INVALID_ARG: return "CHORD_ERR_INVALID_ARG";
    case CHORD_ERR_UNSUPPORTED: return "CHORD_ERR_UNSUPPORTED";
    case CHORD_ERR_LAYOUT_MISMATCH: return "CHORD_ERR_LAYOUT_MISMATCH";
    case CHORD_ERR_WORKSPACE_TOO_SMALL: return "CHORD_ERR_WORKSPACE_TOO_SMALL";
    case CHORD_ERR_CUDA: return "CHORD_ERR_CUDA";
    case CHORD_ERR_DEVICE: return "CHORD_ERR_DEVICE";
    default: return "CHORD_ERR_UNKNOWN";
  }
}

const char* chord_last_error_detail(void) { return g_detail; }

int64_t chord_moe_align_capacity(int64_t T, int topk, int E, int block_m) {
  if (T < 0 || topk < 1 || E < 1 || block_m < 1) return -1;
  return T * topk + int64_t(E) * (block_m - 1);
}

int64_t chord_moe_align_num_blocks(int64_t T, int topk, int E, int block_m) {
  const int64_t cap = chord_moe_align_capacity(T, topk, E, block_m);
  if (cap < 0) return -1;
  return (cap + block_m - 1) / block_m;
}

size_t chord_moe_align_workspace_bytes(int64_t T, int topk, int E) {
  if (T < 0 || topk < 1 || E < 1) return 0;
  return align_workspace_bytes(T * topk, E);
}

chord_status_t chord_moe_align(const int32_t* topk_ids, int64_t T, int topk, int E, int block_m,
                               int32_t* sorted_ids, int32_t* expert_ids, int32_t* num_tokens_padded,
                               int32_t* expert_offsets, void* workspace, size_t workspace_bytes,
                               chord_stream_t stream) {
  clear_detail();
  chord_status_t st = check_align_args(T, topk, E, block_m);
  if (st != CHORD_OK) return st;
  if ((T > 0 && !topk_ids) || !sorted_ids || !expert_ids || !num_tokens_padded)
    return fail(CHORD_ERR_INVALID_ARG, "null routing pointer");
  const size_t need = align_workspace_bytes(T * topk, E);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(CHORD_ERR_WORKSPACE_TOO_SMALL, "align workspace needs %zu bytes, got %zu", need,
                workspace ? workspace_bytes : size_t(0));
  if (need > 0 && !aligned256(workspace)) return fail(CHORD_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if ((st = current_device(nullptr)) != CHORD_OK) return st;
  const int64_t cap = chord_moe_align_capacity(T, topk, E, block_m);
  const int64_t nblocks = chord_moe_align_num_blocks(T, topk, E, block_m);
  cudaError_t err = launch_align(topk_ids, T * topk, E, block_m, cap, nblocks, sorted_ids,
                                 expert_ids, num_tokens_padded, expert_offsets, workspace,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_align launch");
  return CHORD_OK;
}

chord_status_t chord_router_topk_align(const float* logits, int64_t T, int E_global, int topk, int E,
                                       int block_m, int32_t* topk_ids, float* topk_weights, int32_t* sorted_ids,
                                       int32_t* expert_ids, int32_t* num_tokens_padded, int32_t* expert_offsets,
                                       void* workspace, size_t workspace_bytes, chord_stream_t stream) {
  clear_detail();
  chord_status_t st = check_align_args(T, topk, E, block_m);
  if (st != CHORD_OK) return st;
  if (E_global < topk || E_global > 1024)
    return fail(CHORD_ERR_UNSUPPORTED, "E_global=%d outside [topk=%d, 1024]", E_global, topk);
  if ((T > 0 && (!logits || !topk_ids || !topk_weights)) || !sorted_ids || !expert_ids || !num_tokens_padded)
    return fail(CHORD_ERR_INVALID_ARG, "null routing pointer");
  const size_t need = align_workspace_bytes(T * topk, E);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(CHORD_ERR_WORKSPACE_TOO_SMALL, "align workspace needs %zu bytes, got %zu", need,
                workspace ? workspace_bytes : size_t(0));
  if (need > 0 && !aligned256(workspace)) return fail(CHORD_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if ((st = current_device(nullptr)) != CHORD_OK) return st;
  const int64_t cap = chord_moe_align_capacity(T, topk, E, block_m);
  const int64_t nblocks = chord_moe_align_num_blocks(T, topk, E, block_m);
  cudaError_t err = launch_router_align(logits, T, E_global, topk, topk_ids, topk_weights, E, block_m, cap,
                                        nblocks, sorted_ids, expert_ids, num_tokens_padded, expert_offsets,
                                        workspace, reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "router + moe_align launch");
  return CHORD_OK;
}

size_t chord_repacked_bytes(int E, int N, int K, int group_size) {
  if (E < 1 || N < 1 || K < 1 || group_size != kGroup || N % kTileN || K % kTileK) return 0;
  return size_t(blob_total_bytes(E, N, K));
}

chord_status_t chord_repack_weights(const int32_t* qweight, const uint16_t* scales, int E, int N,
                                    int K, int group_size, int role, void* out, size_t out_bytes,
                                    chord_stream_t stream) {
  clear_detail();
  if (group_size != kGroup)
    return fail(CHORD_ERR_UNSUPPORTED, "group_size=%d; only group-32 scales are supported", group_size);
  if (role < CHORD_ROLE_GATE_UP || role > CHORD_ROLE_GROUPED_MASKED)
    return fail(CHORD_ERR_INVALID_ARG, "role=%d", role);
  if (E < 1 || N < 1 || K < 1) return fail(CHORD_ERR_INVALID_ARG, "E=%d N=%d K=%d", E, N, K);
  if (N % kTileN || K % kTileK)
    return fail(CHORD_ERR_UNSUPPORTED, "N=%d and K=%d must be multiples of 128", N, K);
  if (!qweight || !scales || !out) return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  if (!aligned256(out)) return fail(CHORD_ERR_INVALID_ARG, "output blob not 256-byte aligned");
  const size_t need = size_t(blob_total_bytes(E, N, K));
  if (out_bytes < need) return fail(CHORD_ERR_INVALID_ARG, "blob needs %zu bytes, got %zu", need, out_bytes);
  chord_status_t st;
  if ((st = current_device(nullptr)) != CHORD_OK) return st;
  cudaError_t err = launch_repack(qweight, scales, E, N, K, role, static_cast<uint8_t*>(out),
                                  reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "repack launch");
  std::lock_guard<std::mutex> lk(g_mu);
  g_blobs[out] = BlobInfo{E, N, K, role, need};
  return CHORD_OK;
}

chord_status_t chord_dequant_weights(const void* blob, size_t blob_bytes, uint16_t* w_bf16,
                                     chord_stream_t stream) {
  clear_detail();
  if (!blob || !w_bf16) return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  BlobInfo info;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_blobs.find(blob);
    if (it == g_blobs.end())
      return fail(CHORD_ERR_LAYOUT_MISMATCH, "blob was not prepared by chord_repack_weights in this process");
    info = it->second;
  }
  if (blob_bytes < info.bytes) return fail(CHORD_ERR_INVALID_ARG, "blob_bytes too small");
  chord_status_t st;
  if ((st = current_device(nullptr)) != CHORD_OK) return st;
  cudaError_t err = launch_dequant_blob(static_cast<const uint8_t*>(blob), info.E, info.N, info.K,
                                        info.role, w_bf16, reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "dequant launch");
  return CHORD_OK;
}

int chord_select_block_m(int64_t T, int topk, int E_local, int E_global, int H, int I) {
  if (T < 0 || topk < 1 || E_local < 1 || E_global < E_local) return -1;
  const auto key = std::make_tuple(T, topk, E_local, E_global, H, I);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_select_cache.find(key);
    if (it != g_select_cache.end()) return it->second;
  }
  // expected routed tokens per local expert, without reading the routing back
  const double tok_e = double(T) * topk / double(E_global);
  int bm;
  if (tok_e <= 4.0) bm = 8;
  else if (tok_e <= 10.0) bm = 16;
  else if (tok_e <= 24.0) bm = 32;
  else {
    // tensor-core schedule: one block should hold an expert's rows (the MMA N of an item
    // is its routed rows rounded to 16, so spare capacity costs no MMA work), sized to the
    // expected busiest expert (~1.5x the mean) so the activation ring stages stay small
    const int want = int(tok_e * 1.5 + 15.0) / 16 * 16;
    bm = want < 64 ? 64 : (want > 256 ? 256 : want);
  }
  std::lock_guard<std::mutex> lk(g_mu);
  g_select_cache[key] = bm;
  return bm;
}

size_t chord_moe_workspace_bytes(int64_t T, int topk, int E, int H, int I, int block_m) {
  if (T < 0 || topk < 1 || E < 1 || H < 1 || I < 1 || block_m < 1) return 0;
  return size_t(forward_workspace(T, topk, E, H, I, block_m).total);
}

chord_status_t chord_moe_forward(const uint16_t* hidden, const int32_t* topk_ids,
                                 const float* topk_weights, const int32_t* sorted_ids,
                                 const int32_t* expert_ids, const int32_t* num_tokens_padded,
                                 int block_m, const void* w13, const void* w2, int64_t T, int H,
                                 int I, int E, int topk, uint16_t* out, void* workspace,
                                 size_t workspace_bytes, int flags, chord_stream_t stream_) {
  clear_detail();
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  chord_status_t st = check_align_args(T, topk, E, block_m);
  if (st != CHORD_OK) return st;
  if (H < kTileK || H % kTileK || I < kTileK || I % kTileK)
    return fail(CHORD_ERR_UNSUPPORTED, "H=%d and I=%d must be positive multiples of 128", H, I);
  if ((flags & CHORD_FLAG_FORCE_STREAM) && (flags & CHORD_FLAG_FORCE_TENSOR))
    return fail(CHORD_ERR_INVALID_ARG, "FORCE_STREAM and FORCE_TENSOR are exclusive");
  if (!w13 || !w2 || !workspace || !sorted_ids || !expert_ids || !num_tokens_padded)
    return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  if (T > 0 && (!hidden || !topk_ids || !topk_weights || !out))
    return fail(CHORD_ERR_INVALID_ARG, "null activation pointer");
  if (!aligned256(workspace)) return fail(CHORD_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(CHORD_ERR_INVALID_ARG, "hidden and out must be 16-byte aligned");
  const ForwardWorkspace ws = forward_workspace(T, topk, E, H, I, block_m);
  if (workspace_bytes < ws.total)
    return fail(CHORD_ERR_WORKSPACE_TOO_SMALL, "forward workspace needs %llu bytes, got %zu",
                (unsigned long long)ws.total, workspace_bytes);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto check = [&](const void* p, int role, int N, int K, const char* name) -> chord_status_t {
      auto it = g_blobs.find(p);
      if (it == g_blobs.end()) return CHORD_OK;  // foreign blob: the kernels check its header
      const BlobInfo& b = it->second;
      if (b.role != role || b.E != E || b.N != N || b.K != K)
        return fail(CHORD_ERR_LAYOUT_MISMATCH,
                    "%s blob is role %d [E=%d N=%d K=%d], call needs role %d [E=%d N=%d K=%d]", name,
                    b.role, b.E, b.N, b.K, role, E, N, K);
      return CHORD_OK;
    };
    if ((st = check(w13, CHORD_ROLE_GATE_UP, 2 * I, H, "w13")) != CHORD_OK) return st;
    if ((st = check(w2, CHORD_ROLE_DOWN, H, I, "w2")) != CHORD_OK) return st;
  }
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != CHORD_OK) return st;
  if (T == 0) return CHORD_OK;

  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  ForwardArgs a{};
  a.x = hidden;
  a.topk_ids = topk_ids;
  a.topk_weights = topk_weights;
  a.sorted_ids = sorted_ids;
  a.expert_ids = expert_ids;
  a.ntp = num_tokens_padded;
  a.w13 = static_cast<const uint8_t*>(w13);
  a.w2 = static_cast<const uint8_t*>(w2);
  a.out = out;
  a.a = reinterpret_cast<uint16_t*>(wsb + ws.a_offset);
  a.y = reinterpret_cast<float*>(wsb + ws.y_offset);
  a.xs = reinterpret_cast<uint16_t*>(wsb + ws.xs_offset);
  a.slot_pos = reinterpret_cast<int32_t*>(wsb + ws.slot_pos_offset);
  a.status = reinterpret_cast<uint32_t*>(wsb);
  a.stream_flags = reinterpret_cast<uint32_t*>(wsb + ws.flags_offset);
  a.stream_partial = reinterpret_cast<float*>(wsb + ws.partial_offset);
  a.stream_partial_bytes = ws.partial_bytes;
  a.T = T;
  a.H = H;
  a.I = I;
  a.E = E;
  a.topk = topk;
  a.block_m = block_m;
  a.cap = chord_moe_align_capacity(T, topk, E, block_m);
  a.num_sms = num_sms;

  cudaError_t err;
  if (flags & CHORD_FLAG_VALIDATE_ROUTING) {
    if ((err = launch_validate(a, stream)) != cudaSuccess) return cuda_fail(err, "validate launch");
  }
  const bool timing = g_timing_on;
  cudaEvent_t first = timing ? g_timing[0] : nullptr;
  const bool tensor = (flags & CHORD_FLAG_FORCE_TENSOR) ||
                      (!(flags & CHORD_FLAG_FORCE_STREAM) && block_m > 32);
  a.y_blocked = tensor;
  a.out_f32 = (flags & CHORD_FLAG_OUTPUT_FP32) != 0;
  // early (programmatic) launches on the weight-streaming schedule; not while timing events
  // are recorded between the kernels (an event between two kernels orders them fully)
  a.pdl = !tensor && !timing;
  cudaEvent_t mid = timing ? g_timing[1] : nullptr;
  err = tensor ? launch_tc_gemms(a, stream, first, mid) : launch_stream_gemms(a, stream, first, mid);
  if (err != cudaSuccess) return cuda_fail(err, tensor ? "tensor-core GEMM launch" : "streaming GEMM launch");
  if (timing && (err = record_timing_event(g_timing[2], stream)) != cudaSuccess)
    return cuda_fail(err, "timing event");
  if ((err = launch_combine(a, stream)) != cudaSuccess) return cuda_fail(err, "combine launch");
  if (timing && (err = record_timing_event(g_timing[3], stream)) != cudaSuccess)
    return cuda_fail(err, "timing event");
  return CHORD_OK;
}

size_t chord_grouped_workspace_bytes(int64_t rows, int E) {
  if (rows < 0 || E < 1) return 0;
  return size_t(grouped_workspace(rows, E).total);
}

namespace {

// Shared part of the two grouped entry points: checks, the routing pass, the GEMM.
chord_status_t grouped_gemm(const uint16_t* x, int64_t rows, int K, const int32_t* m_indices,
                            const int32_t* masked_m, int64_t max_m, int64_t expected, const void* w, int E, int N,
                            uint16_t* out, void* workspace, size_t workspace_bytes, int flags, int role,
                            cudaStream_t stream) {
  if (E < 1 || E > 1024) return fail(CHORD_ERR_UNSUPPORTED, "E=%d outside [1, 1024]", E);
  if (K < kTileK || K % kTileK || N < kTileN || N % kTileN)
    return fail(CHORD_ERR_UNSUPPORTED, "N=%d and K=%d must be positive multiples of 128", N, K);
  if (rows < 0 || rows >= (int64_t(1) << 31) - 256)
    return fail(rows < 0 ? CHORD_ERR_INVALID_ARG : CHORD_ERR_UNSUPPORTED, "rows=%lld", (long long)rows);
  if ((flags & CHORD_FLAG_FORCE_STREAM) && (flags & CHORD_FLAG_FORCE_TENSOR))
    return fail(CHORD_ERR_INVALID_ARG, "FORCE_STREAM and FORCE_TENSOR are exclusive");
  if (!w || !workspace) return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  if (rows > 0 && (!x || !out || (!m_indices && !masked_m)))
    return fail(CHORD_ERR_INVALID_ARG, "null activation or routing pointer");
  if (!aligned256(workspace)) return fail(CHORD_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(m_indices)) & 15)
    return fail(CHORD_ERR_INVALID_ARG, "x, out and m_indices must be 16-byte aligned");
  const GroupedWorkspace ws = grouped_workspace(rows, E);
  if (workspace_bytes < size_t(ws.total))
    return fail(CHORD_ERR_WORKSPACE_TOO_SMALL, "grouped workspace needs %llu bytes, got %zu",
                (unsigned long long)ws.total, workspace_bytes);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_blobs.find(w);
    if (it != g_blobs.end()) {  // foreign blobs: the kernels check their header
      const BlobInfo& b = it->second;
      if (b.role != role || b.E != E || b.N != N || b.K != K)
        return fail(CHORD_ERR_LAYOUT_MISMATCH,
                    "weight blob is role %d [E=%d N=%d K=%d], call needs role %d [E=%d N=%d K=%d]", b.role, b.E,
                    b.N, b.K, role, E, N, K);
    }
  }
  chord_status_t st;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != CHORD_OK) return st;
  if (rows == 0) return CHORD_OK;

  // schedule: few rows per expert stream the weights (mma.sync over units of 8, 16 or 32
  // rows, one token chunk each); more go to the tensor cores, with units of 32 to 256 rows
  // sized to the expected rows (a smaller unit leaves room for deeper operand rings)
  const bool tensor = (flags & CHORD_FLAG_FORCE_TENSOR) || (!(flags & CHORD_FLAG_FORCE_STREAM) && expected > 16);
  const int bm = tensor ? (expected <= 32 ? 32 : expected <= 64 ? 64 : expected <= 128 ? 128 : 256)
                        : (expected <= 8 ? 8 : (expected <= 16 ? 16 : 32));
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  GroupedArgs g{};
  g.x = x;
  g.rows = rows;
  g.K = K;
  g.N = N;
  g.E = E;
  g.role = role;
  g.w = static_cast<const uint8_t*>(w);
  g.out = out;
  g.expert_ids = reinterpret_cast<int32_t*>(wsb + ws.expert_ids_offset);
  g.block_row0 = reinterpret_cast<int32_t*>(wsb + ws.block_row0_offset);
  g.sorted_ids = reinterpret_cast<int32_t*>(wsb + ws.sorted_ids_offset);
  g.ntp = reinterpret_cast<int32_t*>(wsb + ws.ntp_offset);
  g.bm = bm;
  g.cap = ws.max_positions;
  g.status = reinterpret_cast<uint32_t*>(wsb);
  g.stream_flags = reinterpret_cast<uint32_t*>(wsb + ws.flags_offset);
  g.stream_partial = reinterpret_cast<float*>(wsb + ws.partial_offset);
  g.num_sms = num_sms;
  cudaError_t err = launch_grouped_route(m_indices, rows, masked_m, E, max_m, bm,
                                         const_cast<int32_t*>(g.expert_ids), const_cast<int32_t*>(g.block_row0),
                                         const_cast<int32_t*>(g.sorted_ids), const_cast<int32_t*>(g.ntp), g.status,
                                         stream);
  if (err != cudaSuccess) return cuda_fail(err, "grouped routing launch");
  const bool timing = g_timing_on;
  if (timing && (err = record_timing_event(g_timing[0], stream)) != cudaSuccess) return cuda_fail(err, "timing event");
  err = tensor ? launch_tc_grouped(g, stream) : launch_stream_grouped(g, stream);
  if (err != cudaSuccess) return cuda_fail(err, tensor ? "tensor-core GEMM launch" : "streaming GEMM launch");
  if (timing && (err = record_timing_event(g_timing[1], stream)) != cudaSuccess) return cuda_fail(err, "timing event");
  return CHORD_OK;
}

}  // namespace

chord_status_t chord_grouped_contiguous(const uint16_t* x, int64_t M, int K, const int32_t* m_indices,
                                        const void* w, int E, int N, uint16_t* out, void* workspace,
                                        size_t workspace_bytes, int flags, chord_stream_t stream) {
  clear_detail();
  if (M < 0) return fail(CHORD_ERR_INVALID_ARG, "M=%lld", (long long)M);
  const int64_t expected = E > 0 ? (M + E - 1) / E : 0;
  return grouped_gemm(x, M, K, m_indices, nullptr, 0, expected, w, E, N, out, workspace, workspace_bytes, flags,
                      CHORD_ROLE_GROUPED_CONTIGUOUS, reinterpret_cast<cudaStream_t>(stream));
}

chord_status_t chord_grouped_masked(const uint16_t* x, int E, int64_t max_m, int K, const int32_t* masked_m,
                                    int64_t expected_m, const void* w, int N, uint16_t* out, void* workspace,
                                    size_t workspace_bytes, int flags, chord_stream_t stream) {
  clear_detail();
  if (max_m < 1 || expected_m < 1)
    return fail(CHORD_ERR_INVALID_ARG, "max_m=%lld expected_m=%lld", (long long)max_m, (long long)expected_m);
  if (E < 1 || E > 1024) return fail(CHORD_ERR_UNSUPPORTED, "E=%d outside [1, 1024]", E);
  if (!masked_m) return fail(CHORD_ERR_INVALID_ARG, "null masked_m");
  return grouped_gemm(x, int64_t(E) * max_m, K, nullptr, masked_m, max_m, expected_m, w, E, N, out, workspace,
                      workspace_bytes, flags, CHORD_ROLE_GROUPED_MASKED, reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------------------------
// Exchange steps of sharded deployments

namespace {

chord_status_t check_ep_args(int64_t T, int topk, int E_rank, int W) {
  if (T < 0 || topk < 1 || topk > 64) return fail(CHORD_ERR_INVALID_ARG, "T=%lld topk=%d", (long long)T, topk);
  if (W < 1 || W > 64) return fail(CHORD_ERR_UNSUPPORTED, "W=%d ranks outside [1, 64]", W);
  if (E_rank < 1 || int64_t(E_rank) * W > 4096)
    return fail(CHORD_ERR_UNSUPPORTED, "E_rank=%d x W=%d experts outside [1, 4096]", E_rank, W);
  if (T >= (int64_t(1) << 31) / W) return fail(CHORD_ERR_UNSUPPORTED, "T*W >= 2^31");
  return CHORD_OK;
}

struct EpPlanWorkspace {
  uint64_t ids_offset, expert_ids_offset, ntp_offset, align_offset, total;
};
EpPlanWorkspace ep_plan_workspace(int64_t T, int W) {
  EpPlanWorkspace w;
  const uint64_t n = uint64_t(T) * W;
  w.ids_offset = 0;
  w.expert_ids_offset = align256(n * 4);
  w.ntp_offset = w.expert_ids_offset + align256(n * 4 > 0 ? n * 4 : 4);
  w.align_offset = w.ntp_offset + 256;
  w.total = w.align_offset + align256(align_workspace_bytes(int64_t(n), W));
  return w;
}

}  // namespace

size_t chord_ep_plan_workspace_bytes(int64_t T, int W) {
  if (T < 0 || W < 1) return 0;
  return size_t(ep_plan_workspace(T, W).total);
}

chord_status_t chord_ep_plan(const int32_t* topk_ids, int64_t T, int topk, int E_rank, int W, int32_t* send_rows,
                             int32_t* rank_offsets, int32_t* row_of, void* workspace, size_t workspace_bytes,
                             chord_stream_t stream) {
  clear_detail();
  chord_status_t st = check_ep_args(T, topk, E_rank, W);
  if (st != CHORD_OK) return st;
  if ((T > 0 && (!topk_ids || !send_rows || !row_of)) || !rank_offsets || !workspace)
    return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  if (!aligned256(workspace)) return fail(CHORD_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  const EpPlanWorkspace ws = ep_plan_workspace(T, W);
  if (workspace_bytes < ws.total)
    return fail(CHORD_ERR_WORKSPACE_TOO_SMALL, "ep plan workspace needs %llu bytes, got %zu",
                (unsigned long long)ws.total, workspace_bytes);
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != CHORD_OK) return st;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  int32_t* ids_tw = reinterpret_cast<int32_t*>(wsb + ws.ids_offset);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err = cudaSuccess;
  if (T > 0) err = launch_ep_route(topk_ids, T, topk, E_rank, W, ids_tw, row_of, num_sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "ep route launch");
  // the routing sort over W "experts" (the ranks) with blocks of one row: rows grouped by
  // destination, ascending token inside each, and the per-rank offsets
  const int64_t n = T * W;
  err = launch_align(ids_tw, n, W, 1, n, n, send_rows ? send_rows : ids_tw,
                     reinterpret_cast<int32_t*>(wsb + ws.expert_ids_offset), reinterpret_cast<int32_t*>(wsb + ws.ntp_offset),
                     rank_offsets, wsb + ws.align_offset, s);
  if (err != cudaSuccess) return cuda_fail(err, "ep plan sort launch");
  return CHORD_OK;
}

chord_status_t chord_ep_pack(const uint16_t* hidden, const int32_t* topk_ids, const float* topk_weights, int64_t T,
                             int H, int topk, int E_rank, int W, const int32_t* send_rows, const int32_t* rank_offsets,
                             int32_t* row_of, uint16_t* send_x, int32_t* send_ids, float* send_w,
                             chord_stream_t stream) {
  clear_detail();
  chord_status_t st = check_ep_args(T, topk, E_rank, W);
  if (st != CHORD_OK) return st;
  if (H < 8 || H % 8) return fail(CHORD_ERR_UNSUPPORTED, "H=%d must be a positive multiple of 8", H);
  if (T == 0) return CHORD_OK;
  if (!hidden || !topk_ids || !topk_weights || !send_rows || !rank_offsets || !row_of || !send_x || !send_ids || !send_w)
    return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(send_x)) & 15)
    return fail(CHORD_ERR_INVALID_ARG, "hidden and send_x must be 16-byte aligned");
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != CHORD_OK) return st;
  const cudaError_t err = launch_ep_pack(hidden, topk_ids, topk_weights, T, H, topk, E_rank, W, send_rows, rank_offsets,
                                         send_x, send_ids, send_w, row_of, num_sms, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? CHORD_OK : cuda_fail(err, "ep pack launch");
}

chord_status_t chord_ep_combine(const uint16_t* back, const int32_t* row_of, int64_t T, int H, int W, uint16_t* out,
                                chord_stream_t stream) {
  clear_detail();
  if (T < 0 || W < 1 || W > 64) return fail(CHORD_ERR_INVALID_ARG, "T=%lld W=%d", (long long)T, W);
  if (H < 8 || H % 8) return fail(CHORD_ERR_UNSUPPORTED, "H=%d must be a positive multiple of 8", H);
  if (T == 0) return CHORD_OK;
  if (!row_of || !out) return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(back) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(CHORD_ERR_INVALID_ARG, "back and out must be 16-byte aligned");
  chord_status_t st;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != CHORD_OK) return st;
  const cudaError_t err =
      launch_ep_combine(back, row_of, T * W, T, H, W, out, num_sms, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? CHORD_OK : cuda_fail(err, "ep combine launch");
}

chord_status_t chord_round_bf16(const float* in, int64_t n, uint16_t* out, chord_stream_t stream) {
  clear_detail();
  if (n < 0) return fail(CHORD_ERR_INVALID_ARG, "n=%lld", (long long)n);
  if (n == 0) return CHORD_OK;
  if (!in || !out) return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  chord_status_t st;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != CHORD_OK) return st;
  const cudaError_t err = launch_round_bf16(in, n, out, num_sms, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? CHORD_OK : cuda_fail(err, "round launch");
}

chord_status_t chord_tp_reduce_round(const float* const* partials, uint16_t* const* outs, int W, int rank, int64_t n,
                                    chord_stream_t stream) {
  clear_detail();
  if (W < 1 || W > kMaxTpRanks || rank < 0 || rank >= W)
    return fail(CHORD_ERR_INVALID_ARG, "W=%d rank=%d (1 <= W <= %d)", W, rank, kMaxTpRanks);
  if (n < 0 || n % 4) return fail(CHORD_ERR_INVALID_ARG, "n=%lld must be a non-negative multiple of 4", (long long)n);
  if (!partials || !outs) return fail(CHORD_ERR_INVALID_ARG, "null pointer array");
  TpPeers peers{};
  for (int s = 0; s < W; ++s) {
    if (!partials[s] || !outs[s]) return fail(CHORD_ERR_INVALID_ARG, "null pointer for rank %d", s);
    if ((reinterpret_cast<uintptr_t>(partials[s]) & 15) || (reinterpret_cast<uintptr_t>(outs[s]) & 7))
      return fail(CHORD_ERR_INVALID_ARG, "rank %d: partials must be 16-byte and outputs 8-byte aligned", s);
    peers.in[s] = partials[s];
    peers.out[s] = outs[s];
  }
  if (n == 0) return CHORD_OK;
  chord_status_t st;
  int num_sms = 0;
  if ((st = current_device(&num_sms)) != CHORD_OK) return st;
  const cudaError_t err = launch_tp_reduce_round(peers, W, rank, n, num_sms, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? CHORD_OK : cuda_fail(err, "tp reduce launch");
}

chord_status_t chord_set_timing_events(void* const* events, int n) {
  clear_detail();
  if (n == 0) {
    g_timing_on = false;
    return CHORD_OK;
  }
  if (n != 4 || !events) return fail(CHORD_ERR_INVALID_ARG, "need exactly 4 events, got %d", n);
  for (int i = 0; i < 4; ++i) {
    if (!events[i]) return fail(CHORD_ERR_INVALID_ARG, "null event %d", i);
    g_timing[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_timing_on = true;
  return CHORD_OK;
}

uint64_t chord_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

chord_status_t chord_selftest_wait_timeout(uint32_t* status, uint64_t* elapsed_ns, uint32_t limit_us,
                                           chord_stream_t stream) {
  clear_detail();
  if (!status || !elapsed_ns) return fail(CHORD_ERR_INVALID_ARG, "null pointer");
  if (limit_us < 1 || limit_us > 1000000u)
    return fail(CHORD_ERR_INVALID_ARG, "limit_us must be in [1, 1000000], got %u", limit_us);
  chord_status_t st = current_device(nullptr);
  if (st != CHORD_OK) return st;
  const cudaError_t err = launch_wait_timeout(status, elapsed_ns, uint64_t(limit_us) * 1000ull,
                                              reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? CHORD_OK : cuda_fail(err, "wait self-test launch");
}

chord_status_t chord_moe_check_status(void* workspace, chord_stream_t stream_, uint32_t* device_status) {
  clear_detail();
  if (!workspace) return fail(CHORD_ERR_INVALID_ARG, "null workspace");
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  uint32_t v = 0;
  cudaError_t err = cudaStreamSynchronize(stream);
  if (err != cudaSuccess) return cuda_fail(err, "cudaStreamSynchronize");
  err = cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost);
  if (err != cudaSuccess) return cuda_fail(err, "status read");
  if (v != 0) {
    err = cudaMemsetAsync(workspace, 0, sizeof v, stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize(stream);
    if (err != cudaSuccess) return cuda_fail(err, "status clear");
  }
  if (device_status) *device_status = v;
  if (v != 0) return fail(CHORD_ERR_DEVICE, "device status 0x%x", v);
  return CHORD_OK;
}

}  // extern "C"
