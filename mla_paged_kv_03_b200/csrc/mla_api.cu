// mla_api.cu -- the C ABI of libmla_b200 (declared in include/mla.h):
// argument validation, TMA descriptor encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/mla.h"
#include "combine_kernel.cuh"
#include "decode_kernel.cuh"
#include "page_kernel.cuh"
#include "pair_kernel.cuh"
#include "prologue_kernel.cuh"
#include "prefill_kernel.cuh"
#include "sparse_gather.cuh"
#include "mla_common.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define MLA_CHECK_ARG(cond, ...)                              \
  do {                                                        \
    if (!(cond)) return fail(MLA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define MLA_CUDA(call)                                                                  \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(MLA_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));        \
  } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- TMA maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 view [rows, 576] with a {64 cols, 64 rows} box, 128-byte swizzle.
int make_latent_map(CUtensorMap* map, const void* base, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(mla::kD), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(mla::kD) * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

// 2-D bf16 view [rows, 576] with a box one row high and 64 wide, 128-byte
// swizzle: the map of the TMA gather4 loads (four named rows per copy).
int make_gather_map(CUtensorMap* map, const void* base, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(mla::kD), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(mla::kD) * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (gather) failed (%d)", (int)r);
  return MLA_OK;
}

// 3-D bf16 view of the same rows: {64 dims, rows, 9 chunks of 64 dims}
// (strides 1152 B and 128 B) with a {64, box_rows, box_chunks} box, 128-byte
// swizzle; one copy lands [box_chunks][box_rows][64 dims] in shared memory.
int make_latent_map3(CUtensorMap* map, const void* base, long long rows, int box_chunks,
                     int box_rows = 64, int row_elems = mla::kD) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(mla::kChunkD), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(row_elems / mla::kChunkD)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_elems) * 2,
                           static_cast<cuuint64_t>(mla::kChunkD) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_chunks)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
  return MLA_OK;
}

struct WsLayout {
  size_t o_off, lse_off, q_off, total;
};

WsLayout dense_ws_layout(int batch, int R, int d_v, int parts) {
  WsLayout w{};
  const size_t splits = static_cast<size_t>(batch) + parts;
  w.o_off = 0;
  w.lse_off = align_up(splits * R * d_v * sizeof(float), 256);
  w.total = w.lse_off + align_up(splits * R * sizeof(float), 256);
  return w;
}

// Fused decode workspace: the dense layout (d_v 576), then the normalised,
// rotated query rows [batch * R, 576] bf16 that the prologue kernel writes.
WsLayout fused_ws_layout(int batch, int R, int parts) {
  WsLayout w = dense_ws_layout(batch, R, mla::kD, parts);
  w.q_off = align_up(w.total, 256);
  w.total = w.q_off + align_up(static_cast<size_t>(batch) * R * mla::kD * 2, 256);
  return w;
}

// Sparse decode workspace: the gathered bf16 rows (a dense paged buffer of
// pages_per_pair pages per (sequence, query) pair), its block table and
// lengths, the split tables, then the dense decode workspace.
struct SparseWs {
  size_t rows_off, bt_off, len_off, meta_off, splits_off, dense_off, dense_bytes, q_off, total;
  int pages_per_pair;
};

// Workspace of the sparse paths: the compacted bf16 rows, their identity
// block table and lengths, the planner's output, the dense path's own
// workspace and, for the 528-byte rows, the query widened to 576 dims.
SparseWs sparse_ws_layout(int pairs, int topk, int R, int d_v, int parts, bool v41 = false,
                          bool fused = false) {
  SparseWs w{};
  w.pages_per_pair = mla::ceil_div(topk, mla::kPage);
  const size_t pages = static_cast<size_t>(pairs) * w.pages_per_pair;
  w.rows_off = 0;
  w.bt_off = align_up(pages * mla::kPage * mla::kD * 2, 256);
  w.len_off = w.bt_off + align_up(pages * 4, 256);
  w.meta_off = w.len_off + align_up(static_cast<size_t>(pairs) * 4, 256);
  w.splits_off = w.meta_off + align_up(static_cast<size_t>(parts) * mla::kMetaInts * 4, 256);
  w.dense_off = w.splits_off + align_up((static_cast<size_t>(pairs) + 1) * 4, 256);
  w.dense_bytes = fused ? fused_ws_layout(pairs, R, parts).total
                        : dense_ws_layout(pairs, R, d_v, parts).total;
  w.q_off = w.dense_off + align_up(w.dense_bytes, 256);
  w.total = v41 ? w.q_off + align_up(static_cast<size_t>(pairs) * R * mla::kD * 2, 256)
                : w.dense_off + w.dense_bytes;
  return w;
}

// Launch configuration with programmatic dependent launch: the kernel may
// be scheduled before the preceding grid of the stream has finished and
// waits for it in its first instruction (griddepcontrol.wait).
struct PdlLaunch {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  PdlLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x = 1) {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (cluster_x > 1) {
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = cluster_x;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      cfg.numAttrs = 2;
    }
    cfg.attrs = attr;
  }
};

int launch_combine(const mla::CombineParams& cp, bool fused, cudaStream_t st) {
  const long long rows = static_cast<long long>(cp.seq_list ? cp.list_len : cp.batch) * cp.R;
  if (rows == 0) return MLA_OK;
  // few rows (fewer warps than a few per SM): a CTA per row, warps share its splits
  mla::CombineParams c = cp;
  int num_sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  c.row_per_cta = rows < 8LL * num_sms ? 1 : 0;
  const long long ctas = c.row_per_cta ? rows : (rows + mla::kCombineWarps - 1) / mla::kCombineWarps;
  // two splits per iteration when one wave at two CTAs per SM holds the grid
  const bool pairs = ctas <= 2LL * num_sms;
  PdlLaunch L(dim3(static_cast<unsigned>(ctas)), dim3(mla::kCombineThreads), 0, st);
  if (fused && pairs)
    MLA_CUDA(cudaLaunchKernelEx(&L.cfg, mla::mla_combine_kernel<true, true>, c));
  else if (fused)
    MLA_CUDA(cudaLaunchKernelEx(&L.cfg, mla::mla_combine_kernel<true, false>, c));
  else if (pairs)
    MLA_CUDA(cudaLaunchKernelEx(&L.cfg, mla::mla_combine_kernel<false, true>, c));
  else
    MLA_CUDA(cudaLaunchKernelEx(&L.cfg, mla::mla_combine_kernel<false, false>, c));
  return MLA_OK;
}

// Debug slot trace set by mla_set_slot_trace (per host thread).  The sparse
// paths trace their gather and switch the trace off (TraceOff) around the
// dense decode they run over the compacted rows.
thread_local int32_t* t_trace = nullptr;
thread_local long long t_trace_cap = 0;

struct TraceOff {
  int32_t* saved;
  TraceOff() : saved(t_trace) { t_trace = nullptr; }
  ~TraceOff() { t_trace = saved; }
};

// q . k chunks of the CTA-pair kernel for the dense decode a sparse path runs
// internally (0: the 576-dim latent); the V4.1 paths set 8 around that call,
// passing their 512-wide query as it is.
thread_local int t_qk_chunks = 0;

struct QkChunks {
  int saved;
  explicit QkChunks(int n) : saved(t_qk_chunks) { t_qk_chunks = n; }
  ~QkChunks() { t_qk_chunks = saved; }
};

int check_trace(long long entries_per_plane) {
  if (!t_trace) return MLA_OK;
  MLA_CHECK_ARG(t_trace_cap >= 2 * entries_per_plane,
                "slot trace holds %lld entries, the call needs %lld", t_trace_cap,
                2 * entries_per_plane);
  return MLA_OK;
}

// Events set by mla_set_kernel_events (per host thread), recorded around the
// attention kernel of each decode entry point.
thread_local cudaEvent_t t_kernel_start = nullptr;
thread_local cudaEvent_t t_kernel_stop = nullptr;

// Inside a stream capture an event is recorded as an event-record node of the
// graph (cudaEventRecordExternal), so that its replay can be timed.
int record_event(cudaEvent_t ev, cudaStream_t st) {
  if (!ev) return MLA_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  MLA_CUDA(cudaStreamIsCapturing(st, &cs));
  if (cs == cudaStreamCaptureStatusActive)
    MLA_CUDA(cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal));
  else
    MLA_CUDA(cudaEventRecord(ev, st));
  return MLA_OK;
}

int record_start(cudaStream_t st) { return record_event(t_kernel_start, st); }

int record_stop(cudaStream_t st) { return record_event(t_kernel_stop, st); }

// 1-CTA kernel (tokens on M = 128, V re-read for PV) for 33..64 query rows per
// CTA, d_v 576 and the fused variant.
template <int kMode>
int launch_decode(const CUtensorMap& tq, const CUtensorMap& tkv, const mla::DecodeParams& p,
                  cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(mla::mla_decode_kernel<kMode>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    mla::cfg::kSmemBytes);
  });
  if (attr_err != cudaSuccess)
    return fail(MLA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  int rc = MLA_OK;
  const unsigned grid = static_cast<unsigned>(p.num_parts * p.n_groups);
  if ((rc = record_start(st)) != MLA_OK) return rc;
  PdlLaunch L(dim3(grid), dim3(mla::Threads<kMode>::value), mla::cfg::kSmemBytes, st);
  MLA_CUDA(cudaLaunchKernelEx(&L.cfg, mla::mla_decode_kernel<kMode>, tq, tkv, p));
  return record_stop(st);
}

// Page-resident kernel for up to 32 query rows per KV head (d_v 512).
int launch_page_decode(const void* q, const CUtensorMap& tkv, const mla::DecodeParams& p,
                       cudaStream_t st) {
  using Cfg = mla::PageCfg;
  CUtensorMap tq3;
  int rc = make_latent_map3(&tq3, q, static_cast<long long>(p.batch) * p.R, mla::kNumChunks,
                            Cfg::kRows);
  if (rc != MLA_OK) return rc;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(mla::mla_page_decode_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  });
  if (attr_err != cudaSuccess)
    return fail(MLA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  PdlLaunch L(dim3(static_cast<unsigned>(p.num_parts * p.n_groups)), dim3(Cfg::kThreads),
              Cfg::kSmemBytes, st);
  if ((rc = record_start(st)) != MLA_OK) return rc;
  MLA_CUDA(cudaLaunchKernelEx(&L.cfg, mla::mla_page_decode_kernel, tq3, tkv, p));
  return record_stop(st);
}

// 2-CTA kernel for more than 64 query rows per KV head: clusters of two CTAs,
// one pair per scheduler part and 128-row group.
// In gather mode tkv is the gather map of the row array and no V map is used.
template <bool kGather>
int launch_pair_decode(const void* q, const void* kcache, const CUtensorMap& tkv,
                       const mla::DecodeParams& p, cudaStream_t st) {
  CUtensorMap tq3, tv3;
  // q is [rows, 64 * qk_chunks] (576 wide, or 512 for a 512-dim latent)
  const int qk = p.qk_chunks ? p.qk_chunks : mla::kNumChunks;
  int rc = make_latent_map3(&tq3, q, static_cast<long long>(p.batch) * p.R, qk, 64,
                            qk * mla::kChunkD);
  if (rc != MLA_OK) return rc;
  if (kGather)
    tv3 = tkv;
  else if ((rc = make_latent_map3(&tv3, kcache, static_cast<long long>(p.num_blocks) * mla::kPage,
                                  2)) != MLA_OK)
    return rc;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(mla::mla_pair_decode_kernel<kGather>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    mla::pcfg::kSmemBytes);
  });
  if (attr_err != cudaSuccess)
    return fail(MLA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(attr_err));
  PdlLaunch L(dim3(static_cast<unsigned>(2 * p.num_parts * p.n_groups)), dim3(mla::pcfg::kThreads),
              mla::pcfg::kSmemBytes, st, 2);
  if ((rc = record_start(st)) != MLA_OK) return rc;
  MLA_CUDA(cudaLaunchKernelEx(&L.cfg, mla::mla_pair_decode_kernel<kGather>, tq3, tkv, tv3, p));
  return record_stop(st);
}

int check_common_dense(const void* q, const void* kcache, const int32_t* block_table,
                       int max_pages, int num_blocks, const int32_t* cache_seqlens, int batch,
                       int h_q, float softmax_scale, const int32_t* metadata,
                       const int32_t* num_splits, int num_sm_parts, void* workspace) {
  MLA_CHECK_ARG(batch >= 0, "batch must be >= 0 (got %d)", batch);
  MLA_CHECK_ARG(h_q >= 1, "h_q must be >= 1 (got %d)", h_q);
  MLA_CHECK_ARG(num_sm_parts >= 1 && num_sm_parts <= mla::kCombineMaxSplits,
                "num_sm_parts must be in [1, %d] (got %d)", mla::kCombineMaxSplits, num_sm_parts);
  MLA_CHECK_ARG(max_pages >= 1 && static_cast<long long>(max_pages) * mla::kPage < (1LL << 31),
                "max_pages must be in [1, 2^31 / 64) (got %d)", max_pages);
  MLA_CHECK_ARG(num_blocks >= 1, "num_blocks must be >= 1 (got %d)", num_blocks);
  MLA_CHECK_ARG(static_cast<long long>(num_blocks) * mla::kPage < (1LL << 31),
                "num_blocks * 64 must fit in int32");
  MLA_CHECK_ARG(std::isfinite(softmax_scale) && softmax_scale > 0.f,
                "softmax_scale must be finite and > 0");
  MLA_CHECK_ARG(q && kcache && block_table && cache_seqlens && metadata && num_splits && workspace,
                "null device pointer argument");
  MLA_CHECK_ARG(aligned(q, 16) && aligned(kcache, 16), "q and kcache must be 16-byte aligned");
  MLA_CHECK_ARG(aligned(workspace, 16), "workspace must be 16-byte aligned");
  MLA_CHECK_ARG(aligned(block_table, 4) && aligned(cache_seqlens, 4) && aligned(metadata, 4) &&
                    aligned(num_splits, 4),
                "int32 arrays must be 4-byte aligned");
  return MLA_OK;
}

// Every argument check of mla_decode_fwd (nothing is launched).
int check_dense_decode(const void* q, const void* kcache, const int32_t* block_table,
                       int max_pages, int num_blocks, const int32_t* cache_seqlens, int batch,
                       int s_q, int h_q, int h_kv, int d_v, float softmax_scale,
                       const int32_t* metadata, const int32_t* num_splits, int num_sm_parts,
                       void* workspace, size_t workspace_bytes, void* out, float* lse) {
  if (h_kv != 1) return fail(MLA_ERR_UNSUPPORTED, "h_kv must be 1 (got %d)", h_kv);
  MLA_CHECK_ARG(s_q >= 1, "s_q must be >= 1 (got %d)", s_q);
  MLA_CHECK_ARG(d_v == 512 || d_v == 576, "d_v must be 512 or 576 (got %d)", d_v);
  int rc = check_common_dense(q, kcache, block_table, max_pages, num_blocks, cache_seqlens, batch,
                              h_q, softmax_scale, metadata, num_splits, num_sm_parts, workspace);
  if (rc != MLA_OK) return rc;
  MLA_CHECK_ARG(out && lse, "null output pointer");
  MLA_CHECK_ARG(aligned(out, 16) && aligned(lse, 4), "out must be 16-byte aligned, lse 4-byte");
  const WsLayout w = dense_ws_layout(batch, s_q * h_q, d_v, num_sm_parts);
  MLA_CHECK_ARG(workspace_bytes >= w.total, "workspace too small: %zu < %zu", workspace_bytes,
                w.total);
  return check_trace(static_cast<long long>(batch) * max_pages * mla::kPage);
}

// ------------------------------------------------- fixed-scratch decode
//
// Some callers cannot hand the library a workspace: an embedder whose device
// memory is owned by another allocator (every byte pre-reserved for the KV
// cache pool), or code that must not call an allocator at the moment it
// decodes.  mla_decode_fwd_noalloc serves them from one scratch array that
// lives in the library's own device image.  Every call on a device shares the
// array, so calls whose work may overlap on the GPU (different streams, no
// ordering between them) race on it; callers order them on one stream.
// Nothing in the array needs to start at zero: the planner writes the split
// tables and the decode kernel writes every partial the combine reads.

constexpr size_t kStaticScratchBytes = static_cast<size_t>(32) << 20;
constexpr int kStaticScratchMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device.  The first call
// on a device looks the symbol up (once, with that device current); later
// calls read the cached pointer.
int static_scratch_ptr(void** ptr) {
  int dev = -1;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kStaticScratchMaxDevices)
    return fail(MLA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kStaticScratchMaxDevices);
  static std::mutex mu;
  static void* table[kStaticScratchMaxDevices] = {};
  std::lock_guard<std::mutex> lk(mu);
  if (!table[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return fail(MLA_ERR_CUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev,
                  cudaGetErrorString(e));
    table[dev] = p;
  }
  *ptr = table[dev];
  return MLA_OK;
}

}  // namespace

// Both sparse paths: gather + dequantise + compact the valid rows of every
// (sequence, query) pair, then the dense planner and decode over them.
// Sparse paths, first half: gather + dequantise + compact the valid tokens of
// every (sequence, query) pair into the workspace (rows, identity block table,
// lengths; for the 512-dim V4.1 rows also the query widened to 576 dims,
// returned in *q_dense), then the planner over those lengths.
static int sparse_gather_and_plan(int row_bytes, const void* q, const uint8_t* kcache,
                                  int64_t num_slots, const int32_t* indices, int topk, int pairs,
                                  int h_q, int num_sm_parts, uint8_t* ws, const SparseWs& w,
                                  void* stream, const void** q_dense,
                                  int32_t* trace = nullptr,
                                  long long trace_plane = 0, bool widen_q = true) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  mla::GatherParams g{};
  g.trace = trace;
  g.trace_plane = trace_plane;
  g.cache = kcache;
  g.num_slots = num_slots;
  g.indices = indices;
  g.topk = topk;
  g.pages_per_pair = w.pages_per_pair;
  g.rows = reinterpret_cast<__nv_bfloat16*>(ws + w.rows_off);
  g.block_table = reinterpret_cast<int32_t*>(ws + w.bt_off);
  g.seqlens = reinterpret_cast<int32_t*>(ws + w.len_off);
  g.h_q = h_q;
  *q_dense = q;
  if ((row_bytes == mla::kRow528 || row_bytes == mla::kRow288) && widen_q) {
    g.q512 = static_cast<const __nv_bfloat16*>(q);
    g.q576 = reinterpret_cast<__nv_bfloat16*>(ws + w.q_off);
    *q_dense = g.q576;
  }
  const dim3 grid(w.pages_per_pair, pairs);
  if (row_bytes == mla::kRow528) {
    mla::mla_sparse_gather_kernel<mla::kRow528><<<grid, mla::kGatherCtaThreads, 0, st>>>(g);
  } else if (row_bytes == mla::kRow288) {
    mla::mla_sparse_gather_kernel<mla::kRow288><<<grid, mla::kGatherCtaThreads, 0, st>>>(g);
  } else {
    mla::mla_sparse_gather_kernel<mla::kRow656><<<grid, mla::kGatherCtaThreads, 0, st>>>(g);
  }
  MLA_CUDA(cudaGetLastError());
  return mla_get_metadata(g.seqlens, pairs, h_q, 1, num_sm_parts,
                          reinterpret_cast<int32_t*>(ws + w.meta_off),
                          reinterpret_cast<int32_t*>(ws + w.splits_off), stream);
}

static int sparse_decode_impl(int row_bytes, const void* q, const uint8_t* kcache, int64_t num_slots,
                       const int32_t* indices, int topk, int batch, int s_q, int h_q, int d_v,
                       float softmax_scale, int num_sm_parts, void* workspace,
                       size_t workspace_bytes, void* out, float* lse, void* stream) {
  const bool v41 = row_bytes != mla::kRow656;  // 512-dim latent: query widened to 576
  MLA_CHECK_ARG(batch >= 0 && s_q >= 1 && h_q >= 1, "bad sizes");
  MLA_CHECK_ARG(topk >= 1, "topk must be >= 1 (got %d)", topk);
  MLA_CHECK_ARG(num_slots >= 1 && num_slots < (1LL << 31), "num_slots must be in [1, 2^31)");
  MLA_CHECK_ARG(d_v == 512, "sparse decode supports d_v = 512 (got %d)", d_v);
  MLA_CHECK_ARG(num_sm_parts >= 1 && num_sm_parts <= mla::kCombineMaxSplits,
                "num_sm_parts must be in [1, %d]", mla::kCombineMaxSplits);
  MLA_CHECK_ARG(std::isfinite(softmax_scale) && softmax_scale > 0.f,
                "softmax_scale must be finite and > 0");
  MLA_CHECK_ARG(q && kcache && indices && workspace && out && lse, "null device pointer");
  MLA_CHECK_ARG(aligned(q, 16) && aligned(kcache, 16), "q and the cache must be 16-byte aligned");
  MLA_CHECK_ARG(aligned(workspace, 256), "workspace must be 256-byte aligned");
  MLA_CHECK_ARG(aligned(out, 8) && aligned(lse, 4) && aligned(indices, 4), "misaligned output");
  const int pairs = batch * s_q;
  MLA_CHECK_ARG(aligned(out, 16), "out must be 16-byte aligned");
  const SparseWs w = sparse_ws_layout(pairs, topk, h_q, d_v, num_sm_parts, v41);
  MLA_CHECK_ARG(workspace_bytes >= w.total, "workspace too small: %zu < %zu", workspace_bytes,
                w.total);
  MLA_CHECK_ARG(pairs <= mla::kPlanMaxBatch, "at most %d (batch, query) pairs (got %d)",
                mla::kPlanMaxBatch, pairs);
  const long long pages = static_cast<long long>(pairs) * w.pages_per_pair;
  MLA_CHECK_ARG(pages * mla::kPage < (1LL << 31), "pairs * topk too large");
  int rc = check_trace(static_cast<long long>(pairs) * topk);
  if (rc != MLA_OK) return rc;
  if (batch == 0) return MLA_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const void* q_dense = q;
  // V4.1 rows with more than 64 query rows per KV head: the CTA-pair kernel
  // takes the 512-wide query as it is and reads 8 chunks of each row; the
  // other kernels see the query widened to 576 dims with zeros
  const bool native512 = v41 && h_q > mla::kRowsPerCta && d_v == 512;
  rc = sparse_gather_and_plan(row_bytes, q, kcache, num_slots, indices, topk, pairs, h_q,
                              num_sm_parts, ws, w, stream, &q_dense, t_trace,
                              static_cast<long long>(pairs) * topk, !native512);
  if (rc != MLA_OK) return rc;
  // dense decode over the compacted rows: no causal mask, lengths = valid counts
  TraceOff off;
  QkChunks qk(native512 ? mla::kNumChunks - 1 : 0);
  return mla_decode_fwd(q_dense, ws + w.rows_off, reinterpret_cast<int32_t*>(ws + w.bt_off),
                        w.pages_per_pair, static_cast<int>(pages),
                        reinterpret_cast<int32_t*>(ws + w.len_off), pairs, 1, h_q, 1, d_v,
                        softmax_scale, 0, reinterpret_cast<int32_t*>(ws + w.meta_off),
                        reinterpret_cast<int32_t*>(ws + w.splits_off), num_sm_parts,
                        ws + w.dense_off, w.dense_bytes, out, lse, stream);
}

namespace {

// Query tokens per launch of the sparse prefill (the device planner's limit).
constexpr int kPrefillPass = mla::kPlanMaxBatch;

// Workspace of the sparse prefill, for one pass of up to kPrefillPass tokens:
// the clamped top-k lengths, the split plan (metadata, num_splits, compact
// partial bases) and the partials of the query tokens split over several
// parts (at most 2 * parts of them).
struct PrefillWs {
  size_t len_off, meta_off, splits_off, base_off, list_off, o_off, lse_off, total;
};

PrefillWs prefill_ws_layout(int tokens, int h_q, int parts) {
  PrefillWs w{};
  const size_t rows = 2 * static_cast<size_t>(parts) * h_q;
  w.len_off = 0;
  w.meta_off = align_up(static_cast<size_t>(tokens) * 4, 256);
  w.splits_off = w.meta_off + align_up(static_cast<size_t>(parts) * mla::kMetaInts * 4, 256);
  w.base_off = w.splits_off + align_up((static_cast<size_t>(tokens) + 1) * 4, 256);
  w.list_off = w.base_off + align_up(static_cast<size_t>(tokens) * 4, 256);
  w.o_off = w.list_off + align_up(static_cast<size_t>(parts) * 4, 256);
  w.lse_off = w.o_off + align_up(rows * 512 * 4, 256);
  w.total = w.lse_off + align_up(rows * 4, 256);
  return w;
}

// CTA-pair parts of the prefill launch: at most the caller's count, and no
// more pairs than the device has SMs for.
int prefill_parts(int num_sm_parts, int h_q, int* parts) {
  int dev = 0, sms = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  MLA_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int groups = mla::ceil_div(h_q, 2 * mla::kRowsPerCta);
  const int cap = sms / (2 * groups);
  *parts = num_sm_parts < cap ? num_sm_parts : cap;
  if (*parts < 1) *parts = 1;
  return MLA_OK;
}

}  // namespace

extern "C" {

size_t mla_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

int mla_decode_fwd_noalloc(const void* q, const void* kcache, const int32_t* block_table,
                           int max_pages, int num_blocks, const int32_t* cache_seqlens, int batch,
                           int s_q, int h_q, int h_kv, int d_v, float softmax_scale, int causal,
                           void* out, float* lse, void* stream) {
  if (h_kv != 1) return fail(MLA_ERR_UNSUPPORTED, "h_kv must be 1 (got %d)", h_kv);
  MLA_CHECK_ARG(batch >= 0, "batch must be >= 0 (got %d)", batch);
  MLA_CHECK_ARG(s_q >= 1 && h_q >= 1, "s_q and h_q must be >= 1");
  MLA_CHECK_ARG(d_v == 512 || d_v == 576, "d_v must be 512 or 576 (got %d)", d_v);
  MLA_CHECK_ARG(batch <= mla::kPlanMaxBatch, "at most %d sequences (got %d)", mla::kPlanMaxBatch,
                batch);
  // the caller's pointers first (the scratch ones are checked with the rest below)
  MLA_CHECK_ARG(q && kcache && block_table && cache_seqlens && out && lse,
                "null device pointer argument");
  MLA_CHECK_ARG(aligned(q, 16) && aligned(kcache, 16) && aligned(out, 16),
                "q, kcache and out must be 16-byte aligned");
  MLA_CHECK_ARG(aligned(block_table, 4) && aligned(cache_seqlens, 4) && aligned(lse, 4),
                "block_table, cache_seqlens and lse must be 4-byte aligned");
  int dev = -1;
  MLA_CUDA(cudaGetDevice(&dev));
  const int R = s_q * h_q;
  int parts = 0;
  int rc = mla_num_sm_parts(dev, R, h_kv, &parts);
  if (rc != MLA_OK) return rc;
  // [metadata parts x 8 int32 | num_splits batch+1 int32 | decode workspace]
  const size_t meta_bytes = align_up(static_cast<size_t>(parts) * mla::kMetaInts * 4, 256);
  const size_t splits_bytes = align_up((static_cast<size_t>(batch) + 1) * 4, 256);
  const size_t ws_bytes = dense_ws_layout(batch, R, d_v, parts).total;
  const size_t need = meta_bytes + splits_bytes + ws_bytes;
  if (need > kStaticScratchBytes)
    return fail(MLA_ERR_INVALID_ARG,
                "mla_decode_fwd_noalloc: batch %d x %d rows x d_v %d needs %zu scratch bytes, "
                "above the fixed %zu; use mla_decode_fwd with a caller workspace",
                batch, R, d_v, need, kStaticScratchBytes);
  void* base = nullptr;
  if ((rc = static_scratch_ptr(&base)) != MLA_OK) return rc;
  uint8_t* b8 = static_cast<uint8_t*>(base);
  int32_t* metadata = reinterpret_cast<int32_t*>(b8);
  int32_t* num_splits = reinterpret_cast<int32_t*>(b8 + meta_bytes);
  void* ws = b8 + meta_bytes + splits_bytes;
  // every check of the decode call, before the planner writes the shared array
  if ((rc = check_dense_decode(q, kcache, block_table, max_pages, num_blocks, cache_seqlens, batch,
                               s_q, h_q, h_kv, d_v, softmax_scale, metadata, num_splits, parts, ws,
                               ws_bytes, out, lse)) != MLA_OK)
    return rc;
  if (batch == 0) return MLA_OK;
  if ((rc = mla_get_metadata(cache_seqlens, batch, R, h_kv, parts, metadata, num_splits,
                             stream)) != MLA_OK)
    return rc;
  return mla_decode_fwd(q, kcache, block_table, max_pages, num_blocks, cache_seqlens, batch, s_q,
                        h_q, h_kv, d_v, softmax_scale, causal, metadata, num_splits, parts, ws,
                        ws_bytes, out, lse, stream);
}


const char* mla_last_error(void) { return g_err.c_str(); }

int mla_num_sms(int device, int* num_sms) {
  MLA_CHECK_ARG(num_sms, "num_sms is null");
  int v = 0;
  MLA_CUDA(cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device));
  *num_sms = v;
  return MLA_OK;
}

int mla_num_sm_parts(int device, int heads_per_kv, int h_kv, int* num_sm_parts) {
  MLA_CHECK_ARG(num_sm_parts, "num_sm_parts is null");
  MLA_CHECK_ARG(heads_per_kv >= 1, "heads_per_kv must be >= 1");
  if (h_kv != 1) return fail(MLA_ERR_UNSUPPORTED, "h_kv must be 1 (got %d)", h_kv);
  int sms = 0;
  int rc = mla_num_sms(device, &sms);
  if (rc != MLA_OK) return rc;
  const int groups = mla::ceil_div(heads_per_kv, mla::kRowsPerCta);
  int parts = sms / groups / h_kv;
  *num_sm_parts = parts < 1 ? 1 : parts;
  return MLA_OK;
}

int mla_metadata_size(int batch, int num_sm_parts, size_t* metadata_bytes,
                      size_t* num_splits_bytes) {
  MLA_CHECK_ARG(batch >= 0 && num_sm_parts >= 1, "batch >= 0 and num_sm_parts >= 1 required");
  MLA_CHECK_ARG(metadata_bytes && num_splits_bytes, "null out-pointer");
  *metadata_bytes = static_cast<size_t>(num_sm_parts) * mla::kMetaInts * sizeof(int32_t);
  *num_splits_bytes = (static_cast<size_t>(batch) + 1) * sizeof(int32_t);
  return MLA_OK;
}

int mla_get_metadata(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv,
                     int num_sm_parts, int32_t* metadata, int32_t* num_splits, void* stream) {
  MLA_CHECK_ARG(batch >= 0 && num_sm_parts >= 1, "batch >= 0 and num_sm_parts >= 1 required");
  MLA_CHECK_ARG(heads_per_kv >= 1, "heads_per_kv must be >= 1");
  if (h_kv != 1) return fail(MLA_ERR_UNSUPPORTED, "h_kv must be 1 (got %d)", h_kv);
  MLA_CHECK_ARG(metadata && num_splits && (cache_seqlens || batch == 0), "null device pointer");
  MLA_CHECK_ARG(batch <= mla::kPlanMaxBatch, "the device planner takes at most %d sequences (got %d)",
                mla::kPlanMaxBatch, batch);
  mla::mla_plan_kernel<<<1, mla::kPlanThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      cache_seqlens, batch, num_sm_parts, mla::plan_params(heads_per_kv), metadata, num_splits,
      nullptr, nullptr, 0);
  MLA_CUDA(cudaGetLastError());
  return MLA_OK;
}

int mla_get_metadata_host(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv,
                          int num_sm_parts, int32_t* metadata, int32_t* num_splits) {
  MLA_CHECK_ARG(batch >= 0 && num_sm_parts >= 1, "batch >= 0 and num_sm_parts >= 1 required");
  MLA_CHECK_ARG(heads_per_kv >= 1, "heads_per_kv must be >= 1");
  if (h_kv != 1) return fail(MLA_ERR_UNSUPPORTED, "h_kv must be 1 (got %d)", h_kv);
  MLA_CHECK_ARG(metadata && num_splits && (cache_seqlens || batch == 0), "null host pointer");
  for (int b = 0; b < batch; ++b)
    MLA_CHECK_ARG(cache_seqlens[b] >= 0, "cache_seqlens[%d] = %d is negative", b, cache_seqlens[b]);
  const mla::PlanParams pp = mla::plan_params(heads_per_kv);
  std::vector<int32_t> granules(static_cast<size_t>(batch));
  long long total = 0;
  for (int b = 0; b < batch; ++b) {
    granules[b] = mla::granules_of(cache_seqlens[b], pp.g);
    total += pp.o + static_cast<long long>(mla::kPlanTileCost) * pp.g * granules[b];
  }
  MLA_CHECK_ARG(total <= mla::kPlanMaxTotal, "total planner cost %lld above %lld", total,
                mla::kPlanMaxTotal);
  std::vector<int32_t> prefix(static_cast<size_t>(batch) + 1);
  mla::plan_splits_host(granules.data(), batch, num_sm_parts, pp, metadata, num_splits,
                        prefix.data());
  return MLA_OK;
}

int mla_workspace_size(int batch, int rows_per_kv, int d_v, int num_sm_parts, size_t* bytes) {
  MLA_CHECK_ARG(bytes, "bytes is null");
  MLA_CHECK_ARG(batch >= 0 && rows_per_kv >= 1 && num_sm_parts >= 1, "bad sizes");
  MLA_CHECK_ARG(d_v == 512 || d_v == 576, "d_v must be 512 or 576 (got %d)", d_v);
  *bytes = dense_ws_layout(batch, rows_per_kv, d_v, num_sm_parts).total;
  return MLA_OK;
}

int mla_fused_workspace_size(int batch, int h_q, int num_sm_parts, size_t* bytes) {
  MLA_CHECK_ARG(bytes, "bytes is null");
  MLA_CHECK_ARG(batch >= 0 && h_q >= 1 && num_sm_parts >= 1, "bad sizes");
  *bytes = fused_ws_layout(batch, h_q, num_sm_parts).total;
  return MLA_OK;
}

int mla_decode_fwd(const void* q, const void* kcache, const int32_t* block_table, int max_pages,
                   int num_blocks, const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                   int h_kv, int d_v, float softmax_scale, int causal, const int32_t* metadata,
                   const int32_t* num_splits, int num_sm_parts, void* workspace,
                   size_t workspace_bytes, void* out, float* lse, void* stream) {
  int rc = check_dense_decode(q, kcache, block_table, max_pages, num_blocks, cache_seqlens, batch,
                              s_q, h_q, h_kv, d_v, softmax_scale, metadata, num_splits,
                              num_sm_parts, workspace, workspace_bytes, out, lse);
  if (rc != MLA_OK) return rc;
  const int R = s_q * h_q;
  const WsLayout w = dense_ws_layout(batch, R, d_v, num_sm_parts);
  if (batch == 0) return MLA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  CUtensorMap tkv;
  if ((rc = make_latent_map(&tkv, kcache, static_cast<long long>(num_blocks) * mla::kPage)) !=
      MLA_OK)
    return rc;

  mla::DecodeParams p{};
  p.batch = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.R = R;
  p.d_v = d_v;
  p.n_groups = mla::ceil_div(R, mla::kRowsPerCta);
  p.num_parts = num_sm_parts;
  p.num_blocks = num_blocks;
  p.max_pages = max_pages;
  p.causal = causal ? 1 : 0;
  p.always_partial = 0;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.block_table = block_table;
  p.kcache = static_cast<const uint8_t*>(kcache);
  p.seqlens = cache_seqlens;
  p.metadata = metadata;
  p.num_splits = num_splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.o_off);
  p.ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.lse_off);
  p.trace = t_trace;
  p.trace_plane = static_cast<long long>(batch) * max_pages * mla::kPage;
  p.qk_chunks = t_qk_chunks;
  if (t_qk_chunks && !(R > mla::kRowsPerCta && d_v == 512))
    return fail(MLA_ERR_UNSUPPORTED, "a 512-wide query needs the CTA-pair kernel");
  if (R <= 32 && d_v == 512) {
    p.n_groups = 1;
    rc = launch_page_decode(q, tkv, p, st);
  } else if (R > mla::kRowsPerCta && d_v == 512) {
    p.n_groups = mla::ceil_div(R, 2 * mla::kRowsPerCta);
    rc = launch_pair_decode<false>(q, kcache, tkv, p, st);
  } else {
    CUtensorMap tq;
    if ((rc = make_latent_map(&tq, q, static_cast<long long>(batch) * R)) != MLA_OK) return rc;
    rc = launch_decode<mla::kDense>(tq, tkv, p, st);
  }
  if (rc != MLA_OK) return rc;

  mla::CombineParams cp{};
  cp.batch = batch;
  cp.R = R;
  cp.d_v = d_v;
  cp.h_q = h_q;
  cp.num_splits = num_splits;
  cp.ws_o = p.ws_o;
  cp.ws_lse = p.ws_lse;
  cp.out = p.out;
  cp.lse = lse;
  return launch_combine(cp, false, st);
}

int mla_fused_norm_rope_attn_rope_cast(
    const void* q_raw, const float* norm_gain, float eps, float rope_base,
    const int32_t* positions, const void* kcache, const int32_t* block_table, int max_pages,
    int num_blocks, const int32_t* cache_seqlens, int batch, int h_q, float softmax_scale,
    const int32_t* metadata, const int32_t* num_splits, int num_sm_parts, void* workspace,
    size_t workspace_bytes, uint8_t* out_e4m3, float* out_scale, float* lse, void* stream) {
  int rc = check_common_dense(q_raw, kcache, block_table, max_pages, num_blocks, cache_seqlens,
                              batch, h_q, softmax_scale, metadata, num_splits, num_sm_parts,
                              workspace);
  if (rc != MLA_OK) return rc;
  MLA_CHECK_ARG(norm_gain && out_e4m3 && out_scale && lse, "null pointer argument");
  MLA_CHECK_ARG(aligned(norm_gain, 16), "norm_gain must be 16-byte aligned");
  MLA_CHECK_ARG(aligned(out_e4m3, 4) && aligned(out_scale, 4) && aligned(lse, 4),
                "outputs must be 4-byte aligned");
  MLA_CHECK_ARG(std::isfinite(eps) && eps >= 0.f, "eps must be finite and >= 0");
  MLA_CHECK_ARG(std::isfinite(rope_base) && rope_base > 0.f, "rope_base must be > 0");
  const int R = h_q;
  const int d_v = mla::kD;
  const WsLayout w = fused_ws_layout(batch, R, num_sm_parts);
  MLA_CHECK_ARG(workspace_bytes >= w.total, "workspace too small: %zu < %zu", workspace_bytes,
                w.total);
  if ((rc = check_trace(static_cast<long long>(batch) * max_pages * mla::kPage)) != MLA_OK)
    return rc;
  if (batch == 0) return MLA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  CUtensorMap tkv;
  if ((rc = make_latent_map(&tkv, kcache, static_cast<long long>(num_blocks) * mla::kPage)) !=
      MLA_OK)
    return rc;

  mla::DecodeParams p{};
  p.batch = batch;
  p.s_q = 1;
  p.h_q = h_q;
  p.R = R;
  p.d_v = d_v;
  p.n_groups = mla::ceil_div(R, mla::kRowsPerCta);
  p.num_parts = num_sm_parts;
  p.num_blocks = num_blocks;
  p.max_pages = max_pages;
  p.causal = 0;
  p.always_partial = 1;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.block_table = block_table;
  p.kcache = static_cast<const uint8_t*>(kcache);
  p.seqlens = cache_seqlens;
  p.metadata = metadata;
  p.num_splits = num_splits;
  p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.o_off);
  p.ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.lse_off);
  p.trace = t_trace;
  p.trace_plane = static_cast<long long>(batch) * max_pages * mla::kPage;

  // prologue: Q RMSNorm + RoPE, once per row, into the workspace
  mla::FusedQParams fq{};
  fq.q_raw = static_cast<const __nv_bfloat16*>(q_raw);
  fq.gain = norm_gain;
  fq.eps = eps;
  fq.positions = positions;
  fq.seqlens = cache_seqlens;
  fq.rows = batch * R;
  fq.R = R;
  for (int k = 0; k < mla::kRope / 2; ++k)
    fq.inv_freq[k] = std::pow(static_cast<double>(rope_base), -2.0 * k / mla::kRope);
  fq.q_out = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + w.q_off);
  // an ordinary launch: the prologue reads the caller's inputs, which the
  // preceding work of the stream may still be writing
  mla::mla_fused_q_kernel<<<static_cast<unsigned>(mla::ceil_div(fq.rows, mla::kPrologueWarps)),
                            32 * mla::kPrologueWarps, 0, st>>>(fq);
  MLA_CUDA(cudaGetLastError());
  CUtensorMap tq;
  if ((rc = make_latent_map(&tq, fq.q_out, static_cast<long long>(batch) * R)) != MLA_OK)
    return rc;
  rc = launch_decode<mla::kFused>(tq, tkv, p, st);
  if (rc != MLA_OK) return rc;

  mla::CombineParams cp{};
  cp.batch = batch;
  cp.R = R;
  cp.d_v = d_v;
  cp.h_q = h_q;
  cp.num_splits = num_splits;
  cp.ws_o = p.ws_o;
  cp.ws_lse = p.ws_lse;
  cp.lse = lse;
  cp.out_fp8 = out_e4m3;
  cp.out_scale = out_scale;
  cp.seqlens = cache_seqlens;
  cp.positions = positions;
  for (int k = 0; k < mla::kRope / 2; ++k) cp.inv_freq[k] = fq.inv_freq[k];
  return launch_combine(cp, true, st);
}

int mla_sparse_workspace_size(int batch, int s_q, int h_q, int topk, int d_v, int num_sm_parts,
                              size_t* bytes) {
  MLA_CHECK_ARG(bytes, "bytes is null");
  MLA_CHECK_ARG(batch >= 0 && s_q >= 1 && h_q >= 1 && topk >= 1 && num_sm_parts >= 1,
                "bad sizes");
  MLA_CHECK_ARG(d_v == 512, "sparse decode supports d_v = 512 (got %d)", d_v);
  *bytes = sparse_ws_layout(batch * s_q, topk, h_q, d_v, num_sm_parts).total;
  return MLA_OK;
}

int mla_sparse_v41_workspace_size(int batch, int s_q, int h_q, int topk, int num_sm_parts,
                                  size_t* bytes) {
  MLA_CHECK_ARG(bytes, "bytes is null");
  MLA_CHECK_ARG(batch >= 0 && s_q >= 1 && h_q >= 1 && topk >= 1 && num_sm_parts >= 1,
                "bad sizes");
  *bytes = sparse_ws_layout(batch * s_q, topk, h_q, 512, num_sm_parts, true).total;
  return MLA_OK;
}

int mla_sparse_decode(const void* q, const uint8_t* kcache_fp8, int64_t num_slots,
                      const int32_t* indices, int topk, int batch, int s_q, int h_q, int d_v,
                      float softmax_scale, int num_sm_parts, void* workspace,
                      size_t workspace_bytes, void* out, float* lse, void* stream) {
  return sparse_decode_impl(mla::kRow656, q, kcache_fp8, num_slots, indices, topk, batch, s_q, h_q,
                            d_v, softmax_scale, num_sm_parts, workspace, workspace_bytes, out, lse,
                            stream);
}

int mla_sparse_prefill_workspace_size(int s_q, int h_q, int topk, int num_sm_parts,
                                      size_t* bytes) {
  MLA_CHECK_ARG(bytes, "bytes is null");
  MLA_CHECK_ARG(s_q >= 0 && h_q >= 1 && topk >= 1 && num_sm_parts >= 1, "bad sizes");
  const int tokens = s_q < kPrefillPass ? (s_q > 0 ? s_q : 1) : kPrefillPass;
  *bytes = prefill_ws_layout(tokens, h_q, num_sm_parts).total;
  return MLA_OK;
}

int mla_sparse_prefill_fwd(const void* q, const void* kv, int64_t s_kv, const int32_t* indices,
                           int topk, const int32_t* topk_length, const float* attn_sink, int s_q,
                           int h_q, int d_v, float softmax_scale, int num_sm_parts,
                           void* workspace, size_t workspace_bytes, void* out, float* lse,
                           void* stream) {
  MLA_CHECK_ARG(s_q >= 0 && h_q >= 1, "bad sizes");
  MLA_CHECK_ARG(topk >= 1, "topk must be >= 1 (got %d)", topk);
  MLA_CHECK_ARG(s_kv >= 1 && s_kv < (1LL << 31), "s_kv must be in [1, 2^31)");
  MLA_CHECK_ARG(d_v == 512, "sparse prefill supports d_v = 512 (got %d)", d_v);
  MLA_CHECK_ARG(num_sm_parts >= 1 && num_sm_parts <= mla::kCombineMaxSplits,
                "num_sm_parts must be in [1, %d]", mla::kCombineMaxSplits);
  MLA_CHECK_ARG(std::isfinite(softmax_scale) && softmax_scale > 0.f,
                "softmax_scale must be finite and > 0");
  MLA_CHECK_ARG(q && kv && indices && workspace && out && lse, "null device pointer");
  MLA_CHECK_ARG(aligned(q, 16) && aligned(kv, 16) && aligned(out, 16),
                "q, kv and out must be 16-byte aligned");
  MLA_CHECK_ARG(aligned(workspace, 256), "workspace must be 256-byte aligned");
  MLA_CHECK_ARG(aligned(lse, 4) && aligned(indices, 4) && aligned(topk_length, 4) &&
                    aligned(attn_sink, 4),
                "misaligned lse, indices, topk_length or attn_sink");
  const int tokens = s_q < kPrefillPass ? (s_q > 0 ? s_q : 1) : kPrefillPass;
  const PrefillWs w = prefill_ws_layout(tokens, h_q, num_sm_parts);
  MLA_CHECK_ARG(workspace_bytes >= w.total, "workspace too small: %zu < %zu", workspace_bytes,
                w.total);
  const long long trace_plane = static_cast<long long>(s_q) * topk;
  int rc = check_trace(trace_plane);
  if (rc != MLA_OK) return rc;
  if (s_q == 0) return MLA_OK;
  int parts = 0;
  if ((rc = prefill_parts(num_sm_parts, h_q, &parts)) != MLA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* lengths = reinterpret_cast<int32_t*>(ws + w.len_off);
  int32_t* meta = reinterpret_cast<int32_t*>(ws + w.meta_off);
  int32_t* splits = reinterpret_cast<int32_t*>(ws + w.splits_off);
  int32_t* base = reinterpret_cast<int32_t*>(ws + w.base_off);
  int32_t* split_list = reinterpret_cast<int32_t*>(ws + w.list_off);
  if (t_trace) {  // entries no load reaches stay -1
    MLA_CUDA(cudaMemsetAsync(t_trace, 0xFF, 2 * static_cast<size_t>(trace_plane) * 4, st));
  }
  CUtensorMap tkv;
  if ((rc = make_gather_map(&tkv, kv, s_kv)) != MLA_OK) return rc;
  const size_t q_row = static_cast<size_t>(h_q) * mla::kD;  // bf16 values per token
  for (int t0 = 0; t0 < s_q; t0 += kPrefillPass) {
    const int n = s_q - t0 < kPrefillPass ? s_q - t0 : kPrefillPass;
    mla::mla_prefill_lengths_kernel<<<mla::ceil_div(n, 256), 256, 0, st>>>(
        topk_length ? topk_length + t0 : nullptr, topk, n, lengths);
    MLA_CUDA(cudaGetLastError());
    mla::mla_plan_kernel<<<1, mla::kPlanThreads, 0, st>>>(
        lengths, n, parts, mla::plan_params(h_q), meta, splits, base, split_list, parts);
    MLA_CUDA(cudaGetLastError());
    mla::DecodeParams p{};
    p.batch = n;
    p.s_q = 1;
    p.h_q = h_q;
    p.R = h_q;
    p.d_v = d_v;
    p.n_groups = mla::ceil_div(h_q, 2 * mla::kRowsPerCta);
    p.num_parts = parts;
    p.num_blocks = 1;
    p.max_pages = mla::ceil_div(topk, mla::kPage);
    p.causal = 0;
    p.always_partial = 0;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.seqlens = lengths;
    p.metadata = meta;
    p.num_splits = splits;
    p.ws_base = base;
    p.out = static_cast<__nv_bfloat16*>(out) + static_cast<size_t>(t0) * h_q * d_v;
    p.lse = lse + static_cast<size_t>(t0) * h_q;
    p.ws_o = reinterpret_cast<float*>(ws + w.o_off);
    p.ws_lse = reinterpret_cast<float*>(ws + w.lse_off);
    p.gather_idx = indices + static_cast<size_t>(t0) * topk;
    p.gather_stride = topk;
    p.gather_rows = static_cast<int>(s_kv);
    p.trace = t_trace ? t_trace + static_cast<size_t>(t0) * topk : nullptr;
    p.trace_plane = trace_plane;
    p.sink = attn_sink;
    const void* q_t = static_cast<const __nv_bfloat16*>(q) + t0 * q_row;
    if ((rc = launch_pair_decode<true>(q_t, kv, tkv, p, st)) != MLA_OK) return rc;
    mla::CombineParams cp{};
    cp.batch = n;
    cp.R = h_q;
    cp.d_v = d_v;
    cp.h_q = h_q;
    cp.num_splits = splits;
    cp.ws_base = base;
    cp.ws_o = p.ws_o;
    cp.ws_lse = p.ws_lse;
    cp.out = p.out;
    cp.lse = p.lse;
    cp.seq_list = split_list;  // only the tokens split over several parts
    cp.list_len = parts;
    cp.sink = attn_sink;
    if ((rc = launch_combine(cp, false, st)) != MLA_OK) return rc;
  }
  return MLA_OK;
}

int mla_sparse_fused_workspace_size(int batch, int h_q, int topk, int num_sm_parts,
                                    size_t* bytes) {
  MLA_CHECK_ARG(bytes, "bytes is null");
  MLA_CHECK_ARG(batch >= 0 && h_q >= 1 && topk >= 1 && num_sm_parts >= 1, "bad sizes");
  *bytes = sparse_ws_layout(batch, topk, h_q, mla::kD, num_sm_parts, false, true).total;
  return MLA_OK;
}

int mla_sparse_fused_norm_rope_attn_rope_cast(
    const void* q_raw, const float* norm_gain, float eps, float rope_base,
    const int32_t* positions, const uint8_t* kcache_fp8, int64_t num_slots,
    const int32_t* indices, int topk, int batch, int h_q, float softmax_scale, int num_sm_parts,
    void* workspace, size_t workspace_bytes, uint8_t* out_e4m3, float* out_scale, float* lse,
    void* stream) {
  MLA_CHECK_ARG(batch >= 0 && h_q >= 1, "bad sizes");
  MLA_CHECK_ARG(topk >= 1, "topk must be >= 1 (got %d)", topk);
  MLA_CHECK_ARG(num_slots >= 1 && num_slots < (1LL << 31), "num_slots must be in [1, 2^31)");
  MLA_CHECK_ARG(num_sm_parts >= 1 && num_sm_parts <= mla::kCombineMaxSplits,
                "num_sm_parts must be in [1, %d]", mla::kCombineMaxSplits);
  MLA_CHECK_ARG(positions, "positions are required in sparse mode");
  MLA_CHECK_ARG(q_raw && norm_gain && kcache_fp8 && indices && workspace && out_e4m3 &&
                    out_scale && lse,
                "null device pointer");
  MLA_CHECK_ARG(aligned(q_raw, 16) && aligned(kcache_fp8, 16),
                "q_raw and the cache must be 16-byte aligned");
  MLA_CHECK_ARG(aligned(workspace, 256), "workspace must be 256-byte aligned");
  MLA_CHECK_ARG(aligned(indices, 4) && aligned(positions, 4), "misaligned indices or positions");
  const SparseWs w = sparse_ws_layout(batch, topk, h_q, mla::kD, num_sm_parts, false, true);
  MLA_CHECK_ARG(workspace_bytes >= w.total, "workspace too small: %zu < %zu", workspace_bytes,
                w.total);
  MLA_CHECK_ARG(batch <= mla::kPlanMaxBatch, "at most %d sequences (got %d)", mla::kPlanMaxBatch,
                batch);
  const long long pages = static_cast<long long>(batch) * w.pages_per_pair;
  MLA_CHECK_ARG(pages * mla::kPage < (1LL << 31), "batch * topk too large");
  int rc = check_trace(static_cast<long long>(batch) * topk);
  if (rc != MLA_OK) return rc;
  if (batch == 0) return MLA_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const void* q_dense = q_raw;
  rc = sparse_gather_and_plan(mla::kRow656, q_raw, kcache_fp8, num_slots, indices, topk, batch,
                              h_q, num_sm_parts, ws, w, stream, &q_dense, t_trace,
                              static_cast<long long>(batch) * topk);
  if (rc != MLA_OK) return rc;
  // the fused steps over the compacted rows; every query sees all its rows
  TraceOff off;
  return mla_fused_norm_rope_attn_rope_cast(
      q_raw, norm_gain, eps, rope_base, positions, ws + w.rows_off,
      reinterpret_cast<int32_t*>(ws + w.bt_off), w.pages_per_pair, static_cast<int>(pages),
      reinterpret_cast<int32_t*>(ws + w.len_off), batch, h_q, softmax_scale,
      reinterpret_cast<int32_t*>(ws + w.meta_off), reinterpret_cast<int32_t*>(ws + w.splits_off),
      num_sm_parts, ws + w.dense_off, w.dense_bytes, out_e4m3, out_scale, lse, stream);
}

int mla_sparse_decode_v41_fp4(const void* q, const uint8_t* kcache_288, int64_t num_slots,
                              const int32_t* indices, int topk, int batch, int s_q, int h_q,
                              float softmax_scale, int num_sm_parts, void* workspace,
                              size_t workspace_bytes, void* out, float* lse, void* stream) {
  return sparse_decode_impl(mla::kRow288, q, kcache_288, num_slots, indices, topk, batch, s_q, h_q,
                            512, softmax_scale, num_sm_parts, workspace, workspace_bytes, out, lse,
                            stream);
}

int mla_sparse_decode_v41(const void* q, const uint8_t* kcache_528, int64_t num_slots,
                          const int32_t* indices, int topk, int batch, int s_q, int h_q,
                          float softmax_scale, int num_sm_parts, void* workspace,
                          size_t workspace_bytes, void* out, float* lse, void* stream) {
  return sparse_decode_impl(mla::kRow528, q, kcache_528, num_slots, indices, topk, batch, s_q, h_q,
                            512, softmax_scale, num_sm_parts, workspace, workspace_bytes, out, lse,
                            stream);
}


int mla_set_slot_trace(int32_t* trace, int64_t capacity) {
  MLA_CHECK_ARG(!trace || capacity >= 0, "capacity must be >= 0");
  MLA_CHECK_ARG(aligned(trace, 4), "trace must be 4-byte aligned");
  t_trace = trace;
  t_trace_cap = trace ? capacity : 0;
  return MLA_OK;
}

int mla_set_kernel_events(void* start_event, void* stop_event) {
  t_kernel_start = static_cast<cudaEvent_t>(start_event);
  t_kernel_stop = static_cast<cudaEvent_t>(stop_event);
  return MLA_OK;
}

int mla_device_status(int* status, int reset) {
  MLA_CHECK_ARG(status, "status is null");
  MLA_CUDA(cudaDeviceSynchronize());
  int fault = 0, abort_word = 0;
  MLA_CUDA(cudaMemcpyFromSymbol(&fault, mla::ptx::g_status, sizeof(int)));
  MLA_CUDA(cudaMemcpyFromSymbol(&abort_word, mla::ptx::g_abort, sizeof(int)));
  *status = abort_word != 0 ? abort_word : fault;
  if (reset) {
    const int z = 0;
    MLA_CUDA(cudaMemcpyToSymbol(mla::ptx::g_status, &z, sizeof(int)));
    MLA_CUDA(cudaMemcpyToSymbol(mla::ptx::g_abort, &z, sizeof(int)));
  }
  if (abort_word != 0)
    return fail(MLA_ERR_TIMEOUT, "a kernel wait timed out (site 0x%x)", abort_word & 0xFFFF);
  return MLA_OK;
}

}  // extern "C"
