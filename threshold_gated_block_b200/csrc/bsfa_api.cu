// C ABI of the BSFA prefill forward: argument validation, TMA descriptor
// encoding, kernel dispatch and the device status word. The declarations and
// their contracts are in include/bsfa.h.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "bsfa.h"
#ifdef BSFA_TRACE
#include "bsfa_trace.h"
#endif
#include "bsfa_launch.cuh"

namespace {

thread_local char g_last_error[512] = "";

bsfa_status fail(bsfa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

bsfa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BSFA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// One status word per device: kernels OR a nonzero value into it when they give
// up on a bounded wait.
__device__ int g_status_word;
// Per device: V tiles loaded and PV products issued by mask-writing launches.
__device__ unsigned long long g_debug_counts[2];

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
int* g_status_ptr[kMaxDevices] = {};
unsigned long long* g_counts_ptr[kMaxDevices] = {};
int g_cc_major[kMaxDevices] = {};

bsfa_status device_setup(int dev, int** status_ptr, unsigned long long** counts_ptr = nullptr) {
  if (dev < 0 || dev >= kMaxDevices) return fail(BSFA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (g_status_ptr[dev] == nullptr) {
    int major = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    g_cc_major[dev] = major;
    if (major != 10) return fail(BSFA_ERR_UNSUPPORTED, "device %d has compute capability %d.x; sm_100 required", dev, major);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    void* c = nullptr;
    e = cudaGetSymbolAddress(&c, g_debug_counts);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(debug counters)");
    g_counts_ptr[dev] = static_cast<unsigned long long*>(c);
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  if (g_cc_major[dev] != 10) return fail(BSFA_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
  *status_ptr = g_status_ptr[dev];
  if (counts_ptr) *counts_ptr = g_counts_ptr[dev];
  return BSFA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [B, N, H, D] bf16, boxes of 64 (D) x 1 (head) x rows (N) x 1 (batch), 128-byte swizzle.
bool encode_bnhd(CUtensorMap* map, const void* ptr, int B, int N, int H, int D, int rows) {
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)N * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#ifdef BSFA_TRACE
// Trace build only: the device buffer the next launches stamp (see bsfa_trace.h).
unsigned long long* g_trace_buf = nullptr;
int g_trace_ctas = 0;
#endif

// One thread waits, through the same bounded wait the forward kernel uses, on an
// mbarrier that nothing will ever arrive on. The wait gives up after its time
// limit and the kernel reports through the status word, exactly as a forward
// kernel that lost an arrival would.
__global__ void selftest_lost_arrival_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  bsfa::mbar_init(&bar, 1);
  bsfa::fence_mbar_init();
  abort_flag = 0;
  if (!bsfa::mbar_wait(&bar, 0, &abort_flag)) atomicOr(status, 1);
}

}  // namespace

extern "C" {

bsfa_status bsfa_validate(int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal) {
  (void)causal;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || Bq <= 0 || Bk <= 0)
    return fail(BSFA_ERR_INVALID_ARG, "sizes must be positive (B=%d Hq=%d Hkv=%d N=%d D=%d Bq=%d Bk=%d)", B, Hq, Hkv,
                N, D, Bq, Bk);
  if (Hq % Hkv != 0) return fail(BSFA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  if (D != 64 && D != 128) return fail(BSFA_ERR_UNSUPPORTED, "D=%d unsupported (64 or 128)", D);
  if ((Bq != 64 && Bq != 128) || (Bk != 64 && Bk != 128))
    return fail(BSFA_ERR_UNSUPPORTED, "Bq=%d, Bk=%d unsupported (64 or 128)", Bq, Bk);
  const int key_blocks = (int)(((long long)N + Bk - 1) / Bk);
  if (key_blocks > bsfa::kMaxKeyBlocks)
    return fail(BSFA_ERR_UNSUPPORTED, "ceil(N/Bk)=%d exceeds %d key blocks", key_blocks, bsfa::kMaxKeyBlocks);
  const long long rows = (long long)B * N, head_rows = (long long)B * Hq * N;
  if (rows > 0x7fffffffLL || head_rows > 0x7fffffffLL)
    return fail(BSFA_ERR_UNSUPPORTED, "B*Hq*N=%lld exceeds the 32-bit row index", head_rows);
  return BSFA_OK;
}

}  // extern "C"

namespace {

// Every forward entry point: tau_tiles == 0 selects one value per head; gate_gap
// selects the gap gate, tau then holding gamma. With cu_seqlens the input is B
// packed sequences of at most max_seqlen rows in N = total rows.
bsfa_status forward_impl(const void* q, const void* k, const void* v, const float* tau, int tau_tiles, int gate_gap,
                         void* out, float* lse, uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq,
                         int Bk, int causal, void* stream, const int* cu_seqlens = nullptr, int max_seqlen = 0,
                         int kv_begin = 0, int kv_count = -1, int row_begin = 0, int row_end = -1) {
  bsfa_status st;
  if (cu_seqlens) {
    // Packed sequences: the key-block limit (the per-CTA gate decisions) applies
    // to each sequence, i.e. to max_seqlen; the packed total only has to fit the
    // 32-bit row indices.
    if (B <= 0 || max_seqlen <= 0 || N <= 0)
      return fail(BSFA_ERR_INVALID_ARG, "nseq=%d, max_seqlen=%d and total=%d must be positive", B, max_seqlen, N);
    st = bsfa_validate(1, Hq, Hkv, max_seqlen, D, Bq, Bk, causal);
    if (st != BSFA_OK) return st;
    if ((long long)Hq * N > 0x7fffffffLL)
      return fail(BSFA_ERR_UNSUPPORTED, "Hq*total=%lld exceeds the 32-bit row index", (long long)Hq * N);
    if (!aligned(cu_seqlens, 4)) return fail(BSFA_ERR_INVALID_ARG, "cu_seqlens must be 4-byte aligned");
    if ((long long)B * Hq * (((long long)max_seqlen + 127) / 128) > 0x7fffffffLL)
      return fail(BSFA_ERR_UNSUPPORTED, "nseq * Hq * ceil(max_seqlen/128) exceeds the grid");
  } else {
    st = bsfa_validate(B, Hq, Hkv, N, D, Bq, Bk, causal);
    if (st != BSFA_OK) return st;
    max_seqlen = N;
  }
  if (kv_count < 0) kv_count = Hkv;
  if (kv_begin < 0 || kv_count <= 0 || kv_begin + kv_count > Hkv)
    return fail(BSFA_ERR_INVALID_ARG, "KV heads [%d, %d) are not inside [0, %d)", kv_begin, kv_begin + kv_count, Hkv);
  if (row_end < 0) row_end = max_seqlen;
  if (row_begin < 0 || row_begin % 256 != 0 || row_end <= row_begin || row_end > max_seqlen ||
      (cu_seqlens && (row_begin != 0 || row_end != max_seqlen)))
    return fail(BSFA_ERR_INVALID_ARG, "query rows [%d, %d) are not a 256-aligned range inside [0, %d)", row_begin,
                row_end, max_seqlen);
  if (tau_tiles < 0) return fail(BSFA_ERR_INVALID_ARG, "tau_tiles=%d is negative", tau_tiles);
  if (!q || !k || !v || !tau || !out) return fail(BSFA_ERR_INVALID_ARG, "q, k, v, tau and out must be non-null");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return fail(BSFA_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
  if (!aligned(tau, 4) || (lse && !aligned(lse, 4))) return fail(BSFA_ERR_INVALID_ARG, "tau and lse must be 4-byte aligned");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int* status_ptr = nullptr;
  unsigned long long* counts_ptr = nullptr;
  st = device_setup(dev, &status_ptr, &counts_ptr);
  if (st != BSFA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (block_mask) {
    const size_t n = (size_t)B * Hq * (size_t)((max_seqlen + Bq - 1) / Bq) * (size_t)((max_seqlen + Bk - 1) / Bk);
    e = cudaMemsetAsync(block_mask, 3, n, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(block_mask)");
  }

  CUtensorMap tq, tk, tv;
  const int map_b = cu_seqlens ? 1 : B;     // packed sequences are one batch entry of N rows
  if (!encode_bnhd(&tq, q, map_b, N, Hq, D, 128) || !encode_bnhd(&tk, k, map_b, N, Hkv, D, Bk) ||
      !encode_bnhd(&tv, v, map_b, N, Hkv, D, Bk))
    return fail(BSFA_ERR_CUDA, "cuTensorMapEncodeTiled failed");

  bsfa::FwdParams p;
  p.tau = tau;
  p.tau_tiles = tau_tiles;
  p.gate_gap = gate_gap;
  p.cu_seqlens = cu_seqlens;
  p.max_seqlen = max_seqlen;
  p.mask_mq = (max_seqlen + Bq - 1) / Bq;
  p.mask_mkv = (max_seqlen + Bk - 1) / Bk;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.mask = block_mask;
  p.status = status_ptr;
  p.counts = counts_ptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.group = Hq / Hkv;
  // A CTA pairs two query heads of one KV group when the group size is even,
  // otherwise two adjacent 128-row tiles of one head.
  p.pair_heads = (p.group % 2 == 0) ? 1 : 0;
  p.hq_begin = kv_begin * p.group;
  p.hq_count = kv_count * p.group;
  p.trace = nullptr;
  p.trace_ctas = 0;
#ifdef BSFA_TRACE
  p.trace = g_trace_buf;
  p.trace_ctas = g_trace_ctas;
#endif
  p.scale = (float)(1.0 / std::sqrt((double)D));
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  // Row units: 128-row tiles when a CTA pairs two heads, else pairs of adjacent tiles.
  const int unit_rows = p.pair_heads ? 128 : 256;
  p.row_unit0 = row_begin / unit_rows;
  p.row_units = (row_end + unit_rows - 1) / unit_rows - p.row_unit0;
  const int grid = (p.pair_heads ? B * (p.hq_count / 2) : B * p.hq_count) * p.row_units;
  e = (D == 64) ? bsfa::launch_fwd_d64(tq, tk, tv, p, Bq, Bk, causal != 0, block_mask != nullptr, grid, dev, s)
                : bsfa::launch_fwd_d128(tq, tk, tv, p, Bq, Bk, causal != 0, block_mask != nullptr, grid, dev, s);
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return BSFA_OK;
}

// Copy streams and events of the host-buffer path, created once per device and
// reused by every call (so a call allocates nothing). Calls on one device share
// them: each call holds the device's call lock from its first record to its last
// wait, so the events of two calls from different host threads never interleave
// (their copies are serialised).
constexpr int kMaxChunks = 64;
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr, aux = nullptr;   // aux: a second compute stream
  cudaEvent_t start = nullptr, in[kMaxChunks] = {}, done[kMaxChunks] = {}, out = nullptr;
  std::mutex call;
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mutex;

void destroy_pipe_parts(HostPipe& t) {
  if (t.h2d) cudaStreamDestroy(t.h2d);
  if (t.d2h) cudaStreamDestroy(t.d2h);
  if (t.aux) cudaStreamDestroy(t.aux);
  if (t.start) cudaEventDestroy(t.start);
  if (t.out) cudaEventDestroy(t.out);
  for (int c = 0; c < kMaxChunks; ++c) {
    if (t.in[c]) cudaEventDestroy(t.in[c]);
    if (t.done[c]) cudaEventDestroy(t.done[c]);
  }
}

bsfa_status host_pipe(int dev, HostPipe** pipe) {
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe& hp = g_pipe[dev];
  if (hp.h2d == nullptr) {
    // Created into a scratch set and published only when every part exists; on a
    // failure the parts made so far are destroyed and the next call starts over.
    HostPipe t;
    cudaError_t e = cudaStreamCreateWithFlags(&t.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&t.d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&t.aux, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t.start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t.out, cudaEventDisableTiming);
    for (int c = 0; c < kMaxChunks && e == cudaSuccess; ++c) {
      e = cudaEventCreateWithFlags(&t.in[c], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t.done[c], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
      destroy_pipe_parts(t);
      return cuda_fail(e, "creating the copy streams");
    }
    hp.d2h = t.d2h;
    hp.aux = t.aux;
    hp.start = t.start;
    hp.out = t.out;
    for (int c = 0; c < kMaxChunks; ++c) {
      hp.in[c] = t.in[c];
      hp.done[c] = t.done[c];
    }
    hp.h2d = t.h2d;     // last: a non-null h2d marks the set complete
  }
  *pipe = &hp;
  return BSFA_OK;
}

// Rows [r0, r1) of every batch entry of a [B, N, row_bytes] array: one copy
// (B strided pieces of contiguous rows, or one contiguous run when they touch).
cudaError_t copy_rows(void* dst, const void* src, int B, int N, size_t row_bytes, int r0, int r1, cudaMemcpyKind kind,
                      cudaStream_t st) {
  const size_t pitch = (size_t)N * row_bytes;
  if (B == 1 || (r0 == 0 && r1 == N))
    return cudaMemcpyAsync(static_cast<char*>(dst) + (size_t)r0 * row_bytes,
                           static_cast<const char*>(src) + (size_t)r0 * row_bytes,
                           (size_t)(r1 - r0) * row_bytes + (size_t)(B - 1) * pitch, kind, st);
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + (size_t)r0 * row_bytes, pitch,
                           static_cast<const char*>(src) + (size_t)r0 * row_bytes, pitch, (size_t)(r1 - r0) * row_bytes,
                           (size_t)B, kind, st);
}

}  // namespace

extern "C" {

bsfa_status bsfa_forward(const void* q, const void* k, const void* v, const float* tau, void* out, float* lse,
                         uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                         void* stream) {
  return forward_impl(q, k, v, tau, 0, 0, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, stream);
}

bsfa_status bsfa_forward_tau_table(const void* q, const void* k, const void* v, const float* tau_table, int tau_tiles,
                                   void* out, float* lse, uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D,
                                   int Bq, int Bk, int causal, void* stream) {
  if (tau_tiles <= 0) return fail(BSFA_ERR_INVALID_ARG, "tau_tiles=%d must be positive", tau_tiles);
  return forward_impl(q, k, v, tau_table, tau_tiles, 0, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal,
                      stream);
}

bsfa_status bsfa_forward_gap(const void* q, const void* k, const void* v, const float* gamma, void* out, float* lse,
                             uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                             void* stream) {
  return forward_impl(q, k, v, gamma, 0, 1, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, stream);
}

bsfa_status bsfa_forward_heads(const void* q, const void* k, const void* v, const float* tau, void* out, float* lse,
                               uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                               int kv_begin, int kv_count, void* stream) {
  if (kv_begin < 0 || kv_count < 1)
    return fail(BSFA_ERR_INVALID_ARG, "kv_begin=%d, kv_count=%d: need kv_begin >= 0 and kv_count >= 1", kv_begin,
                kv_count);
  return forward_impl(q, k, v, tau, 0, 0, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, stream, nullptr, 0,
                      kv_begin, kv_count);
}

bsfa_status bsfa_forward_rows(const void* q, const void* k, const void* v, const float* tau, void* out, float* lse,
                              uint8_t* block_mask, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk, int causal,
                              int row_begin, int row_end, void* stream) {
  if (row_end < 0) return fail(BSFA_ERR_INVALID_ARG, "row_end=%d is negative", row_end);
  return forward_impl(q, k, v, tau, 0, 0, out, lse, block_mask, B, Hq, Hkv, N, D, Bq, Bk, causal, stream, nullptr, 0,
                      0, -1, row_begin, row_end);
}

bsfa_status bsfa_forward_host(const void* q_host, const void* k_host, const void* v_host, const float* tau_host,
                              void* out_host, float* lse_host, void* q_dev, void* k_dev, void* v_dev, float* tau_dev,
                              void* out_dev, float* lse_dev, int B, int Hq, int Hkv, int N, int D, int Bq, int Bk,
                              int causal, int chunks, void* stream) {
  bsfa_status st = bsfa_validate(B, Hq, Hkv, N, D, Bq, Bk, causal);
  if (st != BSFA_OK) return st;
  if (!q_host || !k_host || !v_host || !tau_host || !out_host || !q_dev || !k_dev || !v_dev || !tau_dev || !out_dev)
    return fail(BSFA_ERR_INVALID_ARG, "host and device q, k, v, tau and out must be non-null");
  if ((lse_host == nullptr) != (lse_dev == nullptr))
    return fail(BSFA_ERR_INVALID_ARG, "lse needs both a host and a device buffer, or neither");
  const int units = (N + 255) / 256;          // chunk boundaries fall on 256-row multiples
  if (chunks < 1 || chunks > units || chunks > kMaxChunks)
    return fail(BSFA_ERR_INVALID_ARG, "chunks=%d must be in [1, min(ceil(N/256)=%d, %d)]", chunks, units, kMaxChunks);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BSFA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  HostPipe* hp = nullptr;
  st = host_pipe(dev, &hp);
  if (st != BSFA_OK) return st;
  std::lock_guard<std::mutex> call_lock(hp->call);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t q_row = (size_t)Hq * D * 2, kv_row = (size_t)Hkv * D * 2;
  // The copies start once earlier work on the caller's stream is done.
  e = cudaEventRecord(hp->start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->h2d, hp->start, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(tau_dev, tau_host, (size_t)Hq * sizeof(float), cudaMemcpyHostToDevice, hp->h2d);
  // K and V go up first, whole (one copy each); then the query rows in chunks,
  // one copy each. A chunk needs its own Q rows and the keys it attends to, all
  // of which have landed by then.
  if (e == cudaSuccess) e = copy_rows(k_dev, k_host, B, N, kv_row, 0, N, cudaMemcpyHostToDevice, hp->h2d);
  if (e == cudaSuccess) e = copy_rows(v_dev, v_host, B, N, kv_row, 0, N, cudaMemcpyHostToDevice, hp->h2d);
  if (e != cudaSuccess) return cuda_fail(e, "host pipeline start");
  int u_prev = 0;
  for (int c = 0; c < chunks; ++c) {
    // Chunk c: query rows [r0, r1) of every batch entry, in whole 256-row units.
    // The chunks shrink towards the end (cumulative share 1 - (1 - (c+1)/chunks)^2,
    // at least one unit each): what is left after the last upload (the last
    // chunk's compute and its copy back) is then short.
    const double f = 1.0 - (1.0 - (double)(c + 1) / chunks) * (1.0 - (double)(c + 1) / chunks);
    int u1 = (c + 1 == chunks) ? units : (int)(units * f + 0.5);
    u1 = std::max(u1, u_prev + 1);
    u1 = std::min(u1, units - (chunks - 1 - c));
    const int r0 = u_prev * 256, r1 = std::min(u1 * 256, N);
    u_prev = u1;
    e = copy_rows(q_dev, q_host, B, N, q_row, r0, r1, cudaMemcpyHostToDevice, hp->h2d);
    if (e == cudaSuccess) e = cudaEventRecord(hp->in[c], hp->h2d);
    // Chunks alternate between the caller's stream and a second compute stream:
    // a late chunk has few CTAs, each as long as the longest causal row, so two
    // of them run side by side.
    cudaStream_t cs = (c % 2 == 0) ? s : hp->aux;
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, hp->in[c], 0);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    st = forward_impl(q_dev, k_dev, v_dev, tau_dev, 0, 0, out_dev, lse_dev, nullptr, B, Hq, Hkv, N, D, Bq, Bk, causal,
                      cs, nullptr, 0, 0, Hkv, r0, r1);
    if (st != BSFA_OK) return st;
    e = cudaEventRecord(hp->done[c], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp->d2h, hp->done[c], 0);
    if (e == cudaSuccess) e = copy_rows(out_host, out_dev, B, N, q_row, r0, r1, cudaMemcpyDeviceToHost, hp->d2h);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  }
  // lse [B, Hq, N] is head-major: a chunk's rows are B * Hq short runs, so it comes
  // back whole, in one copy, behind the last chunk.
  if (lse_host) {
    e = cudaMemcpyAsync(lse_host, lse_dev, (size_t)B * Hq * N * sizeof(float), cudaMemcpyDeviceToHost, hp->d2h);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy (lse)");
  }
  // The caller's stream reaches the end of the call once the last result is on the host.
  e = cudaEventRecord(hp->out, hp->d2h);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hp->out, 0);
  if (e != cudaSuccess) return cuda_fail(e, "host pipeline end");
  return BSFA_OK;
}

bsfa_status bsfa_forward_varlen(const void* q, const void* k, const void* v, const int* cu_seqlens, int nseq,
                                int max_seqlen, const float* tau, void* out, float* lse, uint8_t* block_mask,
                                int total, int Hq, int Hkv, int D, int Bq, int Bk, int causal, void* stream) {
  if (!cu_seqlens) return fail(BSFA_ERR_INVALID_ARG, "cu_seqlens must be non-null");
  return forward_impl(q, k, v, tau, 0, 0, out, lse, block_mask, nseq, Hq, Hkv, total, D, Bq, Bk, causal, stream,
                      cu_seqlens, max_seqlen);
}

bsfa_status bsfa_get_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int* status_ptr = nullptr;
  bsfa_status st = device_setup(dev, &status_ptr);
  if (st != BSFA_OK) return st;
  int word = 0;
  e = cudaMemcpy(&word, status_ptr, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status word)");
  if (word != 0) {
    const int zero = 0;
    e = cudaMemcpy(status_ptr, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(clear status word)");
    return fail(BSFA_ERR_DEVICE_TIMEOUT, "a kernel gave up on a bounded wait (status word 0x%x)", word);
  }
  return BSFA_OK;
}

bsfa_status bsfa_get_debug_counts(void* stream, unsigned long long* v_tiles, unsigned long long* pv_products) {
  if (!v_tiles || !pv_products) return fail(BSFA_ERR_INVALID_ARG, "v_tiles and pv_products must be non-null");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int* status_ptr = nullptr;
  unsigned long long* counts_ptr = nullptr;
  bsfa_status st = device_setup(dev, &status_ptr, &counts_ptr);
  if (st != BSFA_OK) return st;
  unsigned long long h[2] = {0, 0};
  e = cudaMemcpy(h, counts_ptr, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(debug counters)");
  const unsigned long long zero[2] = {0, 0};
  e = cudaMemcpy(counts_ptr, zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(clear debug counters)");
  *v_tiles = h[0];
  *pv_products = h[1];
  return BSFA_OK;
}

bsfa_status bsfa_selftest_lost_arrival(void* stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int* status_ptr = nullptr;
  bsfa_status st = device_setup(dev, &status_ptr);
  if (st != BSFA_OK) return st;
  selftest_lost_arrival_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status_ptr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return BSFA_OK;
}

const char* bsfa_status_string(bsfa_status s) {
  switch (s) {
    case BSFA_OK: return "BSFA_OK";
    case BSFA_ERR_INVALID_ARG: return "BSFA_ERR_INVALID_ARG";
    case BSFA_ERR_UNSUPPORTED: return "BSFA_ERR_UNSUPPORTED";
    case BSFA_ERR_CUDA: return "BSFA_ERR_CUDA";
    case BSFA_ERR_DEVICE_TIMEOUT: return "BSFA_ERR_DEVICE_TIMEOUT";
  }
  return "BSFA_UNKNOWN_STATUS";
}

const char* bsfa_last_error(void) { return g_last_error; }

#ifdef BSFA_TRACE
bsfa_status bsfa_trace_attach(void* buf, int ctas) {
  if (ctas < 0 || (ctas > 0 && buf == nullptr) || !aligned(buf, 8))
    return fail(BSFA_ERR_INVALID_ARG, "trace buffer %p for %d CTAs", buf, ctas);
  g_trace_buf = static_cast<unsigned long long*>(buf);
  g_trace_ctas = ctas;
  return BSFA_OK;
}

int bsfa_trace_stride(void) { return bsfa::kTraceStride; }
#endif

}  // extern "C"
