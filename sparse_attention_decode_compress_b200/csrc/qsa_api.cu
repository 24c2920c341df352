// C-ABI entry points of libqsa.so (declared in include/qsa.h): host-side
// validation, workspace layout and kernel launches.  Every step of the path
// runs in the kernels included below; nothing here touches tensor data.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "qsa.h"
#include "qsa_common.cuh"
#include "compress_append.cuh"
#include "index_topk.cuh"
#include "index_norm.cuh"
#include "prefill.cuh"
#include "sparse_decode.cuh"
#include "sparse_decode_warp.cuh"
#include "sparse_decode_group.cuh"
#include "sparse_decode_streamk.cuh"
#include "sparse_decode_streamk_group.cuh"
#include "lse_merge.cuh"

namespace {

using qsa::CacheDev;

constexpr size_t kAlign = 256;
// Both workspaces start with a header of this many bytes (the layout does
// not depend on the call's sizes).  The chunked decode keeps its work
// counters and split tickets there and zeroes them at the start of every
// call; the indexer leaves it unused (its group maxima and scores follow).
constexpr size_t kTicketBytes = 64 * 1024;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// The indexer's group maxima (one per 2048 / d rows of a request; sized for
// the smallest groups, d = 128), after the workspace header.
size_t index_gmax_bytes(long long B, long long max_blocks) {
  return align_up((size_t)B * (size_t)((max_blocks + 15) / 16) * sizeof(int32_t));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

qsa_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

// Launches a library kernel; `programmatic` sets programmatic stream
// serialisation (every kernel opens with pdl_open(), see qsa_common.cuh).
// Scan, selection, decode and merge take it.  compress_append, which opens
// a decode step, does not: launched early it pulled the next step's
// persistent scan into the tail of the previous step's merge, and steps
// measured ~12% slower on B200.  (Launched early with only the wait, so
// that the scan follows it only when it ends, the 256k step still measured
// ~2 us slower.)
template <typename... KArgs, typename... Args>
qsa_status launch(bool programmatic, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                  cudaStream_t s, Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = programmatic ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  return launch_status();
}

qsa_status check_cache(const qsa_cache *c) {
  if (!c) return QSA_ERR_INVALID_ARG;
  if (c->page_size <= 0 || c->page_size % 4 != 0) return QSA_ERR_INVALID_ARG;
  if (c->num_pages <= 0 || c->num_kv_heads <= 0 || c->max_pages_per_req <= 0)
    return QSA_ERR_INVALID_ARG;
  if (!c->block_table) return QSA_ERR_INVALID_ARG;
  return QSA_OK;
}

CacheDev to_dev(const qsa_cache *c) {
  CacheDev d;
  d.num_pages = c->num_pages;
  d.page_size = c->page_size;
  d.num_kv_heads = c->num_kv_heads;
  d.head_dim = c->head_dim;
  d.idx_dim = c->idx_dim;
  d.kv_dtype = c->kv_dtype;
  d.k_cache = c->k_cache;
  d.v_cache = c->v_cache;
  d.k_scale = c->k_scale;
  d.v_scale = c->v_scale;
  d.kc = c->kc;
  d.ring = c->ring;
  d.ring_rows = c->ring_rows;
  d.block_table = c->block_table;
  d.max_pages_per_req = c->max_pages_per_req;
  d.table_row = nullptr;
  return d;
}

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

int sm_count(int dev) {
  static int cache[kMaxDevices] = {0};
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// Raises a kernel's dynamic shared-memory limit once per device.
template <typename K>
cudaError_t prepare_kernel(K kernel, size_t smem, bool *done_per_device) {
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxDevices && done_per_device[dev]) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done_per_device[dev] = true;
  return e;
}

std::mutex g_mutex;

// ------------------------------------------------------------------ topk --
size_t select_smem() { return sizeof(qsa::topk::SelSmem) + 128; }

template <typename KT, int NTH>
qsa_status launch_select_nth(const qsa::topk::Params &p, cudaStream_t stream) {
  static bool done[kMaxDevices] = {false};
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (prepare_kernel(qsa::topk::select_kernel<KT, NTH>, select_smem(), done) != cudaSuccess)
      return QSA_ERR_CUDA;
  }
  return launch(true, qsa::topk::select_kernel<KT, NTH>, dim3((unsigned)p.B), dim3(NTH), select_smem(),
                stream, p);
}

// The selection, one CTA per request: 1,024 threads, or 512 threads (two
// CTAs per SM: registers and shared memory allow two) for more requests
// than SMs of at most 32,768 blocks, which then take half the waves.  Long
// requests keep 1,024 threads: on the mixed fp8 batch (256 requests of up
// to 262,144 blocks) one wave of 512-thread CTAs took 46 us, two waves of
// 1,024-thread CTAs 39 us; the sparse prefill's 4,096 tokens of ~8,192
// blocks took 156 against 245 us.
constexpr int kSelHalfMaxBlocks = 32768;
template <typename KT>
qsa_status launch_select(const qsa::topk::Params &p, cudaStream_t stream) {
  if (p.B > sm_count(current_device()) && p.max_blocks <= kSelHalfMaxBlocks)
    return launch_select_nth<KT, 512>(p, stream);
  return launch_select_nth<KT, qsa::topk::kSelThreads>(p, stream);
}

// Scan (persistent grid, scores to the buffer) then selection (one CTA per
// request), back to back on the caller's stream.
template <int DI, int BPPC>
qsa_status launch_index_topk(const qsa::topk::Params &p, cudaStream_t stream) {
  using namespace qsa::topk;
  static int blocks_per_sm[kMaxDevices] = {0};
  auto kernel = index_scan_kernel<DI, BPPC>;
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (dev >= 0 && dev < kMaxDevices && !blocks_per_sm[dev]) {
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kScanThreads, 0) != cudaSuccess)
        return QSA_ERR_CUDA;
      blocks_per_sm[dev] = n > 0 ? n : 1;
    }
  }
  const int bps = (dev >= 0 && dev < kMaxDevices) ? blocks_per_sm[dev] : 1;
  const int grid = bps * sm_count(dev);
  qsa_status st = launch(true, kernel, dim3(grid), dim3(kScanThreads), 0, stream, p);
  if (st != QSA_OK) return st;
  return launch_select<IntKeys>(p, stream);
}

// Scan instance for the indexer dim and page geometry: constant page
// geometry for 64- and 16-token pages, any multiple of 16 tokens, and pages
// of 4, 8 or 12 mod 16 tokens (rows of a run may cross a page).
template <int DI>
qsa_status dispatch_index_topk_d(const qsa::topk::Params &p, int P, cudaStream_t s) {
  if (P == 64) return launch_index_topk<DI, 16>(p, s);
  if (P == 16) return launch_index_topk<DI, 4>(p, s);
  if (P % 16 == 0) return launch_index_topk<DI, 0>(p, s);
  return launch_index_topk<DI, -1>(p, s);
}

qsa_status dispatch_index_topk(const qsa::topk::Params &p, int idx_dim, int P, cudaStream_t s) {
  switch (idx_dim) {
    case 32: return dispatch_index_topk_d<32>(p, P, s);
    case 64: return dispatch_index_topk_d<64>(p, P, s);
    default: return dispatch_index_topk_d<128>(p, P, s);
  }
}

// ---------------------------------------------------------------- decode --
// Chunk slots of one (request, kv head) for chunks of `chunk` micro-blocks:
// a split of n entries takes ceil(n / chunk) chunks, so the splits together
// take at most ceil(E / chunk) + S - 1, and the extended list holds at most
// E = topk + 2 entries.
int decode_chunk_slots(int topk, int S, int chunk) {
  return (topk + 2 + chunk - 1) / chunk + S - 1;
}

// Chunk size of the persistent decode: the largest work items that still
// give every worker at most one of them (one wave, no tail of second
// items), within [kMinChunkBlocks, cap].  A (request, kv head) pair gets
// floor(workers / pairs) workers, c = that / S per split; its splits hold
// about (topk + 2) / S entries each, with 20% added for splits that hold
// more than their share, so that each split takes c chunks.  A batch with
// fewer workers than splits takes the largest chunks, and with
// `whole_splits` (a kernel that streams an item in pieces) whole splits:
// one item per split, no chunk merge.  (Two or three smaller chunks per
// warp, balanced through the work counter, measured ~30% slower: each
// chunk's fixed plan / metadata / epilogue latency is paid again.)
int decode_chunk_blocks(int B, int Hkv, int topk, int S, int S_active, long long workers,
                        int cap, bool whole_splits) {
  const long long pairs = (long long)B * Hkv;
  const long long per_split = workers / (pairs > 0 ? pairs : 1) / S_active;
  int chunk = cap;
  if (per_split == 0 && whole_splits) chunk = topk + 2;
  if (per_split > 0) {
    const long long share = ((long long)topk + 2) * 6 / (5 * S);  // split share with 20% headroom
    chunk = (int)std::min<long long>(chunk, (share + per_split - 1) / per_split);
  }
  return std::max(chunk, qsa::dec::kMinChunkBlocks);
}

// Worker warps per SM and ring depth of the persistent warp decode (8 query
// rows per kv head): 12 warps (166 registers, bf16) with a 2-stage ring.
// fp8: 3 or 4 stages (its stages are half the bytes) measured 1.5-3 % slower
// than 2, and 8 warps with 4 stages slower than 12 with 2.
constexpr int kDecWarps = 12;
constexpr int kDecStages = 2;
template <int D, int NT, bool FP8>
qsa_status launch_decode_warp(qsa::dec::Params p, cudaStream_t stream) {
  constexpr int NW = kDecWarps;
  constexpr int NS = kDecStages;
  static bool done[kMaxDevices] = {false};
  static int blocks_per_sm[kMaxDevices] = {0};
  auto kernel = qsa::dec::sparse_decode_warp_kernel<D, NT, FP8, NW, NS>;
  const size_t smem = sizeof(qsa::dec::WarpSmem<D, FP8, NW, NS>) + 128;
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (prepare_kernel(kernel, smem, done) != cudaSuccess) return QSA_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices && !blocks_per_sm[dev]) {
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, NW * 32, smem) != cudaSuccess)
        return QSA_ERR_CUDA;
      blocks_per_sm[dev] = n > 0 ? n : 1;
    }
  }
  const int bps = (dev >= 0 && dev < kMaxDevices) ? blocks_per_sm[dev] : 1;
  const int ctas = bps * sm_count(dev);
  p.chunk = decode_chunk_blocks(p.B, p.c.num_kv_heads, p.topk, p.S, p.s_hi - p.s_lo,
                                (long long)ctas * NW,
                                qsa::dec::warp_piece_blocks<FP8>(), true);
  p.nch = decode_chunk_slots(p.topk, p.S, p.chunk);
  return launch(true, kernel, dim3(ctas), dim3(NW * 32), smem, stream, p);
}

template <int D>
qsa_status launch_decode_f32(qsa::dec::Params p, cudaStream_t stream) {
  static bool done[kMaxDevices] = {false};
  p.chunk = qsa::dec::kMinChunkBlocks;  // one CTA per chunk slot: many small ones
  p.nch = decode_chunk_slots(p.topk, p.S, p.chunk);
  const dim3 grid((unsigned)p.nch, (unsigned)p.c.num_kv_heads, (unsigned)p.B);
  auto kernel = qsa::dec::sparse_decode_f32_kernel<D>;
  const size_t smem = sizeof(qsa::dec::F32Smem<D>) + 128;
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (prepare_kernel(kernel, smem, done) != cudaSuccess) return QSA_ERR_CUDA;
  }
  return launch(true, kernel, grid, dim3(qsa::dec::kThreads), smem, stream, p);
}

// More than 8 query rows: groups of GW = NT warps, one per 8-row tile,
// sharing a ring of NS stages.  bf16: 16 warps per SM (4 groups of 4 at MTP
// verify) with one stage per warp, 128 registers; fp8: 12 warps with two
// stages per warp (at 16 warps its registers spill).  (MTP verify decode:
// 16 warps x 1 stage 63.5 us, 16 x 1.5 65.3 us, 12 x 2 67.1 us.)
template <int D, bool FP8, int GW>
qsa_status launch_decode_group(qsa::dec::Params p, cudaStream_t stream) {
  constexpr int NW = (FP8 ? 12 : 16) / GW * GW;
  constexpr int NS = FP8 ? 2 * GW : GW;
  static bool done[kMaxDevices] = {false};
  static int blocks_per_sm[kMaxDevices] = {0};
  auto kernel = qsa::dec::sparse_decode_group_kernel<D, FP8, NW, NS, GW>;
  const size_t smem = sizeof(qsa::dec::GroupSmem<D, FP8, NW, NS, GW>) + 128;
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (prepare_kernel(kernel, smem, done) != cudaSuccess) return QSA_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices && !blocks_per_sm[dev]) {
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, NW * 32, smem) != cudaSuccess)
        return QSA_ERR_CUDA;
      blocks_per_sm[dev] = n > 0 ? n : 1;
    }
  }
  const int bps = (dev >= 0 && dev < kMaxDevices) ? blocks_per_sm[dev] : 1;
  const int ctas = bps * sm_count(dev);
  p.chunk = decode_chunk_blocks(p.B, p.c.num_kv_heads, p.topk, p.S, p.s_hi - p.s_lo,
                                (long long)ctas * (NW / GW),
                                qsa::dec::kGroupChunkBlocks, false);
  p.nch = decode_chunk_slots(p.topk, p.S, p.chunk);
  return launch(true, kernel, dim3(ctas), dim3(NW * 32), smem, stream, p);
}

// ------------------------------------------------------- stream-K decode --
// Entries per pair in the global list of the stream-K decode; warps of a
// launch (at most 2048, ranges of at least 16 entries; W_hw = the resident
// warps of the device); partial slots per (pair, split): a split of at most
// E entries meets at most ceil(E / l) + 1 warp ranges of l >= floor(X / W)
// entries, largest for the most warps the launch may use (so the workspace
// size needs no device).
int sk_entries(int topk, int T) { return topk + (T > 1 ? 2 : 0); }
constexpr long long kSKMaxWarps = 2048;
constexpr long long kSKMinEntries = 16;
long long sk_warps(long long X, long long w_hw) {
  return std::max<long long>(1, std::min({w_hw, kSKMaxWarps, X / kSKMinEntries}));
}
int sk_slots(long long pairs, int E) {
  const long long X = pairs * E;
  const long long l = X / sk_warps(X, kSKMaxWarps);
  if (l < 1) return 1;  // no entries (B = 0)
  return (int)((E + l - 1) / l) + 1;
}
struct SKLayout {
  size_t ebound, lse, o, total;
};
SKLayout sk_layout(int B, int T, int Hq, int Hkv, int topk, int S, int D) {
  const long long pairs = (long long)B * Hkv;
  const int K = sk_slots(pairs, sk_entries(topk, T));
  const size_t M = (size_t)(Hq / Hkv) * T;
  SKLayout l;
  l.ebound = 0;
  l.lse = align_up((size_t)B * (S + 1) * sizeof(int32_t));
  l.o = l.lse + align_up((size_t)pairs * S * K * M * sizeof(float));
  l.total = l.o + align_up((size_t)pairs * S * K * M * D * sizeof(float));
  return l;
}

// Stream-K decode of bf16 caches and its merge.  GW = 1: one warp per
// worker (at most 8 query rows per kv head); GW = 2..4: groups of GW warps,
// one per 8-row tile, share a worker's ring.
template <int D, int GW>
qsa_status launch_decode_streamk_gw(const qsa::dec::Params &p, float *o, float *lse, void *workspace,
                                    cudaStream_t stream) {
  constexpr int NW = GW == 1 ? kDecWarps : 16 / GW * GW;
  constexpr int NS = GW == 1 ? kDecStages : GW;
  static bool done[kMaxDevices] = {false};
  static int blocks_per_sm[kMaxDevices] = {0};
  auto kernel = []() {
    if constexpr (GW == 1) return qsa::dec::sparse_decode_streamk_kernel<D, NW, NS>;
    else return qsa::dec::sparse_decode_streamk_group_kernel<D, NW, NS, GW>;
  }();
  const size_t smem = (GW == 1 ? sizeof(qsa::dec::WarpSmem<D, false, NW, NS>)
                               : sizeof(qsa::dec::SKGroupSmem<D, NW, NS, GW>)) +
                      128;
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (prepare_kernel(kernel, smem, done) != cudaSuccess) return QSA_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices && !blocks_per_sm[dev]) {
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, NW * 32, smem) != cudaSuccess)
        return QSA_ERR_CUDA;
      blocks_per_sm[dev] = n > 0 ? n : 1;
    }
  }
  const int bps = (dev >= 0 && dev < kMaxDevices) ? blocks_per_sm[dev] : 1;
  constexpr int per_cta = NW / GW;  // workers per CTA
  qsa::dec::SKParams sk;
  sk.p = p;
  sk.p.chunk = 1 << 20;  // the plan's chunk count is not used by these kernels
  const long long pairs = (long long)p.B * p.c.num_kv_heads;
  sk.E = sk_entries(p.topk, p.T);
  sk.X = pairs * sk.E;
  sk.K = sk_slots(pairs, sk.E);
  // one wave of resident CTAs at most; workers past W return at once
  sk.W = (int)sk_warps(sk.X, (long long)bps * sm_count(dev) * per_cta);
  const long long ctas = (sk.W + per_cta - 1) / per_cta;
  const SKLayout lay = sk_layout(p.B, p.T, p.Hq, p.c.num_kv_heads, p.topk, p.S, D);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  sk.sk_ebound = reinterpret_cast<int32_t *>(ws + lay.ebound);
  sk.sk_lse = reinterpret_cast<float *>(ws + lay.lse);
  sk.sk_o = reinterpret_cast<float *>(ws + lay.o);
  sk.o = o;
  sk.lse = lse;
  qsa_status st = launch(true, kernel, dim3((unsigned)ctas), dim3(NW * 32), smem, stream, sk);
  if (st != QSA_OK) return st;
  const long long rows = pairs * p.M;
  const long long grid = (rows * 32 + qsa::dec::kSKMergeThreads - 1) / qsa::dec::kSKMergeThreads;
  if (grid > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  auto merge = (p.s_hi - p.s_lo <= 4) ? qsa::dec::streamk_merge_kernel<D, 4>
                                      : qsa::dec::streamk_merge_kernel<D, qsa::dec::kMaxSplits>;
  return launch(true, merge, dim3((unsigned)grid), dim3(qsa::dec::kSKMergeThreads), 0, stream, sk);
}

template <int D>
qsa_status launch_decode_streamk(const qsa::dec::Params &p, float *o, float *lse, void *workspace,
                                 cudaStream_t stream) {
  switch ((p.M + 7) / 8) {  // 8-row tiles of the query rows
    case 1: return launch_decode_streamk_gw<D, 1>(p, o, lse, workspace, stream);
    case 2: return launch_decode_streamk_gw<D, 2>(p, o, lse, workspace, stream);
    case 3: return launch_decode_streamk_gw<D, 3>(p, o, lse, workspace, stream);
    default: return launch_decode_streamk_gw<D, 4>(p, o, lse, workspace, stream);
  }
}

template <int D, bool FP8>
qsa_status dispatch_decode_nt(const qsa::dec::Params &p, int NT, cudaStream_t stream) {
  switch (NT) {
    case 1: return launch_decode_warp<D, 1, FP8>(p, stream);
    case 2: return launch_decode_group<D, FP8, 2>(p, stream);
    case 3: return launch_decode_group<D, FP8, 3>(p, stream);
    default: return launch_decode_group<D, FP8, 4>(p, stream);
  }
}

template <int D>
qsa_status dispatch_decode_d(const qsa::dec::Params &p, int kv_dtype, cudaStream_t stream) {
  if (kv_dtype == QSA_F32) return launch_decode_f32<D>(p, stream);
  const int NT = (p.M + 7) / 8;  // query rows on the N side, tiles of 8
  if (kv_dtype == QSA_FP8_E4M3) return dispatch_decode_nt<D, true>(p, NT, stream);
  return dispatch_decode_nt<D, false>(p, NT, stream);
}

}  // namespace

extern "C" {

const char *qsa_status_string(int32_t status) {
  switch (status) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG: malformed argument";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED: unsupported shape or dtype";
    case QSA_ERR_BOUNDS: return "QSA_ERR_BOUNDS: page or position out of range";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA: CUDA runtime error";
    case QSA_ERR_TIMEOUT: return "QSA_ERR_TIMEOUT: a bounded device wait ran out";
    case QSA_ERR_BAD_INPUT: return "QSA_ERR_BAD_INPUT: malformed lengths or selection";
    default: return "unknown qsa_status";
  }
}

int32_t qsa_abi_version(void) { return 2; }

size_t qsa_kc_page_bytes(int32_t page_size, int32_t idx_dim) {
  if (page_size <= 0 || page_size % 4 != 0) return 0;
  if (idx_dim != 32 && idx_dim != 64 && idx_dim != 128) return 0;
  return (size_t)qsa::kc_page_bytes(page_size, idx_dim);
}

qsa_status qsa_compress_append(const qsa_cache *cache, int32_t B, const int32_t *pos0,
                               const int32_t *cu_new, const int8_t *k_new,
                               int32_t max_new_per_req, qsa_stream_t stream) {
  qsa_status st = check_cache(cache);
  if (st != QSA_OK) return st;
  if (B < 0 || max_new_per_req < 0) return QSA_ERR_INVALID_ARG;
  if (B == 0 || max_new_per_req == 0) return QSA_OK;
  if (B > cache->ring_rows || B > 65535) return QSA_ERR_INVALID_ARG;
  if (!pos0 || !cu_new || !k_new || !cache->kc || !cache->ring) return QSA_ERR_INVALID_ARG;
  if (!aligned(k_new, 4) || !aligned(cache->kc, 16) || !aligned(cache->ring, 4))
    return QSA_ERR_INVALID_ARG;
  const long long max_blocks = (long long)max_new_per_req / 4 + 2;
  const long long gx = (max_blocks + qsa::kAppendBlocksPerCta - 1) / qsa::kAppendBlocksPerCta;
  if (gx > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  dim3 grid((unsigned)gx, (unsigned)B);
  const CacheDev c = to_dev(cache);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 block(qsa::kAppendThreads);
  switch (cache->idx_dim) {
    case 32: return launch(false, qsa::compress_append_kernel<32>, grid, block, 0, s, c, B, pos0, cu_new, k_new, max_new_per_req);
    case 64: return launch(false, qsa::compress_append_kernel<64>, grid, block, 0, s, c, B, pos0, cu_new, k_new, max_new_per_req);
    case 128: return launch(false, qsa::compress_append_kernel<128>, grid, block, 0, s, c, B, pos0, cu_new, k_new, max_new_per_req);
    default: return QSA_ERR_UNSUPPORTED;
  }
}

size_t qsa_index_topk_workspace_bytes(int32_t B, int32_t max_blocks) {
  if (B < 0 || max_blocks < 0) return 0;
  return kTicketBytes + index_gmax_bytes(B, max_blocks) +
         align_up((size_t)B * (size_t)max_blocks * sizeof(int32_t));
}

}  // extern "C"

namespace {

// Shared body of qsa_index_topk and qsa_index_topk_tokens: validation, then
// scan + selection.  sel and/or tokens receive the output rows.
qsa_status index_topk_call(const qsa_cache *cache, int32_t B, const int8_t *q_idx,
                           const int32_t *ctx_lens, const int32_t *n_sel, int32_t T,
                           int32_t max_blocks, int32_t topk, int32_t *sel, int32_t *tokens,
                           int32_t *scores, void *workspace, size_t workspace_bytes,
                           qsa_stream_t stream) {
  qsa_status st = check_cache(cache);
  if (st != QSA_OK) return st;
  if (B < 0) return QSA_ERR_INVALID_ARG;
  if (topk < 1 || topk > qsa::topk::kMaxTopk) return QSA_ERR_INVALID_ARG;
  if (max_blocks < 1 || max_blocks > (1 << 24)) return QSA_ERR_INVALID_ARG;
  if (T < 1 || T > qsa::dec::kMaxT) return QSA_ERR_INVALID_ARG;
  if (B == 0) return QSA_OK;
  if (B > 0x7fffffff / 2) return QSA_ERR_UNSUPPORTED;
  if (!q_idx || !ctx_lens || !(sel || tokens) || !workspace || !cache->kc) return QSA_ERR_INVALID_ARG;
  if (cache->idx_dim != 32 && cache->idx_dim != 64 && cache->idx_dim != 128)
    return QSA_ERR_UNSUPPORTED;
  if (!aligned(cache->kc, 16) || !aligned(q_idx, 4) || !aligned(workspace, 16) ||
      (scores && !aligned(scores, 4)) || (tokens && !aligned(tokens, 16)))
    return QSA_ERR_INVALID_ARG;
  const size_t gmax_bytes = index_gmax_bytes(B, max_blocks);
  const size_t need = scores ? kTicketBytes + gmax_bytes : qsa_index_topk_workspace_bytes(B, max_blocks);
  if (workspace_bytes < need) return QSA_ERR_INVALID_ARG;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  qsa::topk::Params p;
  p.c = to_dev(cache);
  p.B = B;
  p.q_idx = q_idx;
  p.ctx_lens = ctx_lens;
  p.n_sel = n_sel;
  p.max_blocks = max_blocks;
  p.topk = topk;
  p.sel = sel;
  p.tokens = tokens;
  p.T = T;
  p.scores = scores ? scores : reinterpret_cast<int32_t *>(ws + kTicketBytes + gmax_bytes);
  p.gmax = reinterpret_cast<int32_t *>(ws + kTicketBytes);
  p.gsize = 2048 / cache->idx_dim;
  return dispatch_index_topk(p, cache->idx_dim, cache->page_size,
                             reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

qsa_status qsa_index_topk(const qsa_cache *cache, int32_t B, const int8_t *q_idx,
                          const int32_t *ctx_lens, const int32_t *n_sel, int32_t max_blocks,
                          int32_t topk, int32_t *sel, int32_t *scores, void *workspace,
                          size_t workspace_bytes, qsa_stream_t stream) {
  return index_topk_call(cache, B, q_idx, ctx_lens, n_sel, 1, max_blocks, topk, sel, nullptr,
                         scores, workspace, workspace_bytes, stream);
}

qsa_status qsa_index_topk_tokens(const qsa_cache *cache, int32_t B, const int8_t *q_idx,
                                 const int32_t *ctx_lens, const int32_t *n_sel, int32_t T,
                                 int32_t max_blocks, int32_t budget, int32_t *tokens,
                                 int32_t *sel, int32_t *scores, void *workspace,
                                 size_t workspace_bytes, qsa_stream_t stream) {
  if (budget < 4 || budget % 4 != 0) return QSA_ERR_INVALID_ARG;
  if (B > 0 && !tokens) return QSA_ERR_INVALID_ARG;
  return index_topk_call(cache, B, q_idx, ctx_lens, n_sel, T, max_blocks, budget / 4, sel, tokens,
                         scores, workspace, workspace_bytes, stream);
}

size_t qsa_sparse_decode_workspace_bytes(int32_t B, int32_t T, int32_t Hq, int32_t Hkv,
                                         int32_t D, int32_t topk, int32_t num_splits) {
  if (B < 0 || T < 1 || Hq < 1 || Hkv < 1 || D < 1 || topk < 1 || num_splits < 1) return 0;
  const size_t M = (size_t)(Hq / Hkv) * T;
  // room for the smallest chunks the launch may pick
  const size_t nch = decode_chunk_slots(topk, num_splits, qsa::dec::kMinChunkBlocks);
  const size_t slots = (size_t)B * Hkv * nch;
  const size_t chunked =
      kTicketBytes + align_up(slots * M * D * sizeof(float)) + align_up(slots * M * sizeof(float));
  // the stream-K decode (at most 8 query rows per kv head, bf16 / fp8)
  const size_t streamk = sk_layout(B, T, Hq, Hkv, topk, num_splits, D).total;
  return std::max(chunked, streamk);
}

}  // extern "C"

namespace {

// Shared body of qsa_sparse_decode and qsa_sparse_decode_splits: splits
// [split_lo, split_hi) of num_splits, stored from o_part[0] on.
qsa_status sparse_decode_call(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                              const void *q, int32_t q_dtype, const int32_t *ctx_lens,
                              const int32_t *sel, int32_t topk, float sm_scale, int32_t num_splits,
                              int32_t split_lo, int32_t split_hi, float *o_part, float *lse_part,
                              float *o_merged, float *lse_merged, void *workspace,
                              size_t workspace_bytes, qsa_stream_t stream,
                              const int32_t *table_row = nullptr) {
  qsa_status st = check_cache(cache);
  if (st != QSA_OK) return st;
  const int Hkv = cache->num_kv_heads;
  const int D = cache->head_dim;
  if (B < 0 || T < 1 || Hq < 1 || topk < 1 || topk > qsa::topk::kMaxTopk) return QSA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > qsa::dec::kMaxSplits) return QSA_ERR_INVALID_ARG;
  if (split_lo < 0 || split_hi > num_splits || split_lo >= split_hi) return QSA_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return QSA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return QSA_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (T > qsa::dec::kMaxT || G * T > qsa::dec::kMaxRows) return QSA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return QSA_ERR_UNSUPPORTED;
  if (cache->kv_dtype == QSA_F32) {
    if (q_dtype != QSA_F32) return QSA_ERR_UNSUPPORTED;
  } else if (cache->kv_dtype == QSA_BF16 || cache->kv_dtype == QSA_FP8_E4M3) {
    if (q_dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
  } else {
    return QSA_ERR_UNSUPPORTED;
  }
  if (B == 0) return QSA_OK;
  if (B > 65535 || Hkv > 65535) return QSA_ERR_UNSUPPORTED;
  // cache rows are indexed with 32-bit integers
  if ((long long)cache->num_pages * cache->page_size * Hkv > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  // bf16 caches take the stream-K decode (one warp, or a warp group, per
  // worker); fp8 and fp32 the chunked decode with its ticket header
  const bool streamk = cache->kv_dtype == QSA_BF16;
  if (!streamk && (size_t)B * Hkv * num_splits * sizeof(int32_t) >
                      kTicketBytes - qsa::dec::kCounterInts * sizeof(int32_t))
    return QSA_ERR_UNSUPPORTED;
  const bool merged = o_merged != nullptr;
  if (merged && (!lse_merged || !aligned(o_merged, 16) || split_lo != 0 || split_hi != num_splits))
    return QSA_ERR_INVALID_ARG;
  if (!q || !ctx_lens || !sel || !o_part || !lse_part || !workspace || !cache->k_cache ||
      !cache->v_cache)
    return QSA_ERR_INVALID_ARG;
  if (cache->kv_dtype == QSA_FP8_E4M3 && (!cache->k_scale || !cache->v_scale))
    return QSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(cache->k_cache, 16) || !aligned(cache->v_cache, 16) ||
      !aligned(workspace, 16) || !aligned(o_part, 16))
    return QSA_ERR_INVALID_ARG;
  if (workspace_bytes < qsa_sparse_decode_workspace_bytes(B, T, Hq, Hkv, D, topk, num_splits))
    return QSA_ERR_INVALID_ARG;

  const int nch = decode_chunk_slots(topk, num_splits, qsa::dec::kMinChunkBlocks);
  const int M = G * T;
  qsa::dec::Params p;
  p.c = to_dev(cache);
  p.c.table_row = table_row;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.G = G;
  p.M = M;
  p.q = q;
  p.ctx_lens = ctx_lens;
  p.sel = sel;
  p.topk = topk;
  p.scale_log2 = sm_scale * qsa::dec::kLog2e;
  p.S = num_splits;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.s_lo = split_lo;
  p.s_hi = split_hi;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  p.counters = reinterpret_cast<int32_t *>(ws);
  p.tickets = p.counters + qsa::dec::kCounterInts;

  const size_t slots = (size_t)B * Hkv * nch;
  p.ws_o = reinterpret_cast<float *>(ws + kTicketBytes);
  p.ws_lse = reinterpret_cast<float *>(ws + kTicketBytes + align_up(slots * M * D * sizeof(float)));
  p.nch = nch;  // the launch sets nch and chunk for its kernel
  p.chunk = qsa::dec::kMinChunkBlocks;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (streamk) {
    // decode + merge of its partials (into o_part, and o / lse when merged)
    return D == 64 ? launch_decode_streamk<64>(p, o_merged, lse_merged, workspace, s)
                   : launch_decode_streamk<128>(p, o_merged, lse_merged, workspace, s);
  }
  // the header (work counters, split tickets) starts at zero in every call,
  // whatever the workspace held
  const int header_ints = qsa::dec::kCounterInts + B * Hkv * num_splits;
  st = launch(true, qsa::dec::decode_header_reset_kernel, dim3(1), dim3(1024), 0, s, p.counters,
              header_ints);
  if (st != QSA_OK) return st;
  st = (D == 64) ? dispatch_decode_d<64>(p, cache->kv_dtype, s)
                 : dispatch_decode_d<128>(p, cache->kv_dtype, s);
  // the merge kernel, one warp per output row, right behind the decode
  // (merging inside the decode, by the warp finishing a pair's last split,
  // measured slower: 0.434 against 0.423 ms per 256k step, 0.228 against
  // 0.176 ms per MTP step, from the one warp walking all of a pair's rows)
  if (st != QSA_OK || !merged) return st;
  return qsa_lse_merge(num_splits, (int64_t)B * T * Hq, D, o_part, lse_part, o_merged, lse_merged,
                       stream);
}

}  // namespace

extern "C" {

qsa_status qsa_sparse_decode(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                             const void *q, int32_t q_dtype, const int32_t *ctx_lens,
                             const int32_t *sel, int32_t topk, float sm_scale,
                             int32_t num_splits, float *o_part, float *lse_part,
                             void *workspace, size_t workspace_bytes, qsa_stream_t stream) {
  return sparse_decode_call(cache, B, T, Hq, q, q_dtype, ctx_lens, sel, topk, sm_scale, num_splits,
                            0, num_splits, o_part, lse_part, nullptr, nullptr, workspace,
                            workspace_bytes, stream);
}

qsa_status qsa_sparse_decode_merged(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                                    const void *q, int32_t q_dtype, const int32_t *ctx_lens,
                                    const int32_t *sel, int32_t topk, float sm_scale,
                                    int32_t num_splits, float *o_part, float *lse_part, float *o,
                                    float *lse, void *workspace, size_t workspace_bytes,
                                    qsa_stream_t stream) {
  if (B > 0 && (!o || !lse)) return QSA_ERR_INVALID_ARG;
  return sparse_decode_call(cache, B, T, Hq, q, q_dtype, ctx_lens, sel, topk, sm_scale, num_splits,
                            0, num_splits, o_part, lse_part, o, lse, workspace, workspace_bytes,
                            stream);
}

qsa_status qsa_sparse_decode_splits(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                                    const void *q, int32_t q_dtype, const int32_t *ctx_lens,
                                    const int32_t *sel, int32_t topk, float sm_scale,
                                    int32_t num_splits, int32_t split_lo, int32_t split_hi,
                                    float *o_part, float *lse_part, void *workspace,
                                    size_t workspace_bytes, qsa_stream_t stream) {
  return sparse_decode_call(cache, B, T, Hq, q, q_dtype, ctx_lens, sel, topk, sm_scale, num_splits,
                            split_lo, split_hi, o_part, lse_part, nullptr, nullptr, workspace,
                            workspace_bytes, stream);
}

qsa_status qsa_lse_merge(int32_t num_splits, int64_t rows, int32_t D, const float *o_part,
                         const float *lse_part, float *o, float *lse, qsa_stream_t stream) {
  if (num_splits < 1 || num_splits > qsa::kMergeMaxSplits || rows < 0 || D < 4 || D % 4 != 0)
    return QSA_ERR_INVALID_ARG;
  if (rows == 0) return QSA_OK;
  if (!o_part || !lse_part || !o || !lse) return QSA_ERR_INVALID_ARG;
  if (!aligned(o_part, 16) || !aligned(o, 16) || !aligned(lse_part, 4) || !aligned(lse, 4))
    return QSA_ERR_INVALID_ARG;
  const long long rows_per_cta = qsa::kMergeThreads / 32;
  const long long grid = (rows + rows_per_cta - 1) / rows_per_cta;
  if (grid > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  return launch(true, qsa::lse_merge_kernel, dim3((unsigned)grid), dim3(qsa::kMergeThreads), 0,
                reinterpret_cast<cudaStream_t>(stream), num_splits, rows, D, o_part, lse_part, o, lse);
}

qsa_status qsa_get_device_error(qsa_stream_t stream, uint32_t *flags_out) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return QSA_ERR_CUDA;
  uint32_t flags = 0;
  if (cudaMemcpyFromSymbol(&flags, qsa::g_error_flags, sizeof(flags)) != cudaSuccess)
    return QSA_ERR_CUDA;
  const uint32_t zero = 0;
  if (flags && cudaMemcpyToSymbol(qsa::g_error_flags, &zero, sizeof(zero)) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (flags_out) *flags_out = flags;
  if (flags & qsa::kErrTimeout) return QSA_ERR_TIMEOUT;
  if (flags & qsa::kErrBounds) return QSA_ERR_BOUNDS;
  if (flags & qsa::kErrBadInput) return QSA_ERR_BAD_INPUT;
  return QSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Normalised-pooling indexer (float compressed keys, float scores).
// ---------------------------------------------------------------------------
namespace {

template <int DI>
qsa_status launch_index_topk_norm(const qsa::norm::ScanParams &sp, cudaStream_t stream) {
  using namespace qsa::topk;
  static int blocks_per_sm[kMaxDevices] = {0};
  auto kernel = qsa::norm::index_scan_norm_kernel<DI>;
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (dev >= 0 && dev < kMaxDevices && !blocks_per_sm[dev]) {
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, qsa::norm::kScanThreads, 0) !=
          cudaSuccess)
        return QSA_ERR_CUDA;
      blocks_per_sm[dev] = n > 0 ? n : 1;
    }
  }
  const int bps = (dev >= 0 && dev < kMaxDevices) ? blocks_per_sm[dev] : 1;
  qsa_status st = launch(true, kernel, dim3(bps * sm_count(dev)), dim3(qsa::norm::kScanThreads), 0,
                         stream, sp);
  if (st != QSA_OK) return st;
  return launch_select<FloatKeys>(sp.p, stream);
}

bool norm_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

}  // namespace

extern "C" {

size_t qsa_kcn_page_bytes(int32_t page_size, int32_t idx_dim) {
  if (page_size <= 0 || page_size % 4 != 0 || !norm_dim_ok(idx_dim)) return 0;
  return (size_t)(page_size / 4) * (size_t)idx_dim * 2;
}

qsa_status qsa_compress_append_norm(const qsa_cache *cache, void *kcn, void *ring,
                                    const float *norm_weight, float eps, int32_t B,
                                    const int32_t *pos0, const int32_t *cu_new, const void *k_new,
                                    int32_t max_new_per_req, qsa_stream_t stream) {
  qsa_status st = check_cache(cache);
  if (st != QSA_OK) return st;
  if (B < 0 || max_new_per_req < 0 || !(eps > 0.f) || !std::isfinite(eps)) return QSA_ERR_INVALID_ARG;
  if (!norm_dim_ok(cache->idx_dim)) return QSA_ERR_UNSUPPORTED;
  if (B == 0 || max_new_per_req == 0) return QSA_OK;
  if (B > cache->ring_rows || B > 65535) return QSA_ERR_INVALID_ARG;
  if (!pos0 || !cu_new || !k_new || !kcn || !ring) return QSA_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(kcn, 16) || !aligned(ring, 16) ||
      (norm_weight && !aligned(norm_weight, 4)))
    return QSA_ERR_INVALID_ARG;
  const long long max_blocks = (long long)max_new_per_req / 4 + 2;
  const long long gx = (max_blocks + qsa::norm::kAppendBlocksPerCta - 1) / qsa::norm::kAppendBlocksPerCta;
  if (gx > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  qsa::norm::AppendParams a;
  a.c = to_dev(cache);
  a.kcn = static_cast<__half *>(kcn);
  a.ring = static_cast<__nv_bfloat16 *>(ring);
  a.weight = norm_weight;
  a.eps = eps;
  a.B = B;
  a.pos0 = pos0;
  a.cu_new = cu_new;
  a.k_new = static_cast<const __nv_bfloat16 *>(k_new);
  a.max_new = max_new_per_req;
  const dim3 grid((unsigned)gx, (unsigned)B), block(qsa::norm::kAppendThreads);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (cache->idx_dim) {
    case 32: return launch(false, qsa::norm::compress_append_norm_kernel<32>, grid, block, 0, s, a);
    case 64: return launch(false, qsa::norm::compress_append_norm_kernel<64>, grid, block, 0, s, a);
    default: return launch(false, qsa::norm::compress_append_norm_kernel<128>, grid, block, 0, s, a);
  }
}

qsa_status qsa_index_topk_norm(const qsa_cache *cache, const void *kcn, int32_t B,
                               const void *q_idx, const int32_t *ctx_lens, const int32_t *n_sel,
                               int32_t max_blocks, int32_t topk, int32_t *sel, float *scores,
                               void *workspace, size_t workspace_bytes, qsa_stream_t stream) {
  qsa_status st = check_cache(cache);
  if (st != QSA_OK) return st;
  if (B < 0) return QSA_ERR_INVALID_ARG;
  if (topk < 1 || topk > qsa::topk::kMaxTopk) return QSA_ERR_INVALID_ARG;
  if (max_blocks < 1 || max_blocks > (1 << 24)) return QSA_ERR_INVALID_ARG;
  if (!norm_dim_ok(cache->idx_dim)) return QSA_ERR_UNSUPPORTED;
  if (B == 0) return QSA_OK;
  if (B > 0x7fffffff / 2) return QSA_ERR_UNSUPPORTED;
  if (!kcn || !q_idx || !ctx_lens || !sel || !workspace) return QSA_ERR_INVALID_ARG;
  if (!aligned(kcn, 16) || !aligned(q_idx, 16) || !aligned(workspace, 16) ||
      (scores && !aligned(scores, 4)))
    return QSA_ERR_INVALID_ARG;
  const size_t need = scores ? kTicketBytes : qsa_index_topk_workspace_bytes(B, max_blocks);
  if (workspace_bytes < need) return QSA_ERR_INVALID_ARG;
  qsa::norm::ScanParams sp;
  sp.p.c = to_dev(cache);
  sp.p.B = B;
  sp.p.q_idx = nullptr;
  sp.p.ctx_lens = ctx_lens;
  sp.p.n_sel = n_sel;
  sp.p.max_blocks = max_blocks;
  sp.p.topk = topk;
  sp.p.sel = sel;
  sp.p.scores = scores ? reinterpret_cast<int32_t *>(scores)
                       : reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + kTicketBytes);
  sp.kcn = static_cast<const __half *>(kcn);
  sp.q = static_cast<const __nv_bfloat16 *>(q_idx);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (cache->idx_dim) {
    case 32: return launch_index_topk_norm<32>(sp, s);
    case 64: return launch_index_topk_norm<64>(sp, s);
    default: return launch_index_topk_norm<128>(sp, s);
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Sparse prefill: many query tokens per request, each with its own selection.
// ---------------------------------------------------------------------------
namespace {

struct PrefillLayout {
  size_t scores, tok_len, tok_row, dec, total;
};

PrefillLayout prefill_layout(int32_t n_tokens, int32_t max_blocks, int32_t Hq, int32_t Hkv,
                             int32_t D, int32_t topk) {
  PrefillLayout l;
  l.scores = 0;
  l.tok_len = align_up((size_t)n_tokens * (size_t)max_blocks * sizeof(int32_t));
  l.tok_row = l.tok_len + align_up((size_t)n_tokens * sizeof(int32_t));
  l.dec = l.tok_row + align_up((size_t)n_tokens * sizeof(int32_t));
  l.total = l.dec + qsa_sparse_decode_workspace_bytes(n_tokens, 1, Hq, Hkv, D, topk, 1);
  return l;
}

template <int DI>
qsa_status launch_prefill_scan(const qsa::pre::ScanParams &sp, int B, int max_q, cudaStream_t s) {
  static bool done[kMaxDevices] = {false};
  auto kernel = qsa::pre::prefill_scan_kernel<DI>;
  const size_t smem = qsa::pre::smem_bytes<DI>();
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (prepare_kernel(kernel, smem, done) != cudaSuccess) return QSA_ERR_CUDA;
  }
  const dim3 grid((unsigned)((sp.max_blocks + qsa::pre::kBlkPerCta - 1) / qsa::pre::kBlkPerCta),
                  (unsigned)((max_q + qsa::pre::kTokTile - 1) / qsa::pre::kTokTile), (unsigned)B);
  return launch(true, kernel, grid, dim3(qsa::pre::kThreads), smem, s, sp);
}

}  // namespace

extern "C" {

size_t qsa_sparse_prefill_workspace_bytes(int32_t n_tokens, int32_t max_blocks, int32_t Hq,
                                          int32_t Hkv, int32_t D, int32_t topk) {
  if (n_tokens < 0 || max_blocks < 1 || Hq < 1 || Hkv < 1 || D < 1 || topk < 1) return 0;
  return prefill_layout(n_tokens, max_blocks, Hq, Hkv, D, topk).total;
}

qsa_status qsa_sparse_prefill(const qsa_cache *cache, int32_t B, int32_t n_tokens,
                              int32_t max_q_per_req, const int32_t *cu_q, const int32_t *ctx_lens,
                              const int8_t *q_idx, const int8_t *k_chunk, const void *q,
                              int32_t q_dtype, int32_t Hq, int32_t max_blocks, int32_t topk,
                              float sm_scale, int32_t *sel, float *o, float *lse, void *workspace,
                              size_t workspace_bytes, qsa_stream_t stream) {
  qsa_status st = check_cache(cache);
  if (st != QSA_OK) return st;
  if (B < 0 || n_tokens < 0 || max_q_per_req < 0) return QSA_ERR_INVALID_ARG;
  if (topk < 1 || topk > qsa::topk::kMaxTopk) return QSA_ERR_INVALID_ARG;
  if (max_blocks < 1 || max_blocks > (1 << 24)) return QSA_ERR_INVALID_ARG;
  if (cache->idx_dim != 32 && cache->idx_dim != 64 && cache->idx_dim != 128)
    return QSA_ERR_UNSUPPORTED;
  if (B == 0 || n_tokens == 0) return QSA_OK;
  if (max_q_per_req < 1 || B > 65535 || n_tokens > 65535 ||
      (max_q_per_req + qsa::pre::kTokTile - 1) / qsa::pre::kTokTile > 65535)
    return QSA_ERR_UNSUPPORTED;
  if (!cu_q || !ctx_lens || !q_idx || !k_chunk || !q || !sel || !o || !lse || !workspace ||
      !cache->kc)
    return QSA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(k_chunk, 4) || !aligned(cache->kc, 16) ||
      !aligned(workspace, 256))
    return QSA_ERR_INVALID_ARG;
  const int Hkv = cache->num_kv_heads, D = cache->head_dim;
  if (Hq < 1 || Hq % Hkv != 0) return QSA_ERR_INVALID_ARG;
  const PrefillLayout lay = prefill_layout(n_tokens, max_blocks, Hq, Hkv, D, topk);
  if (workspace_bytes < lay.total) return QSA_ERR_INVALID_ARG;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *scores = reinterpret_cast<int32_t *>(ws + lay.scores);
  int32_t *tok_len = reinterpret_cast<int32_t *>(ws + lay.tok_len);
  int32_t *tok_row = reinterpret_cast<int32_t *>(ws + lay.tok_row);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // 1. scores of every query token against its prefix blocks (tensor cores)
  qsa::pre::ScanParams sp;
  sp.c = to_dev(cache);
  sp.cu_q = cu_q;
  sp.ctx_lens = ctx_lens;
  sp.q_idx = q_idx;
  sp.max_blocks = max_blocks;
  sp.n_tok = n_tokens;
  sp.scores = scores;
  switch (cache->idx_dim) {
    case 32: st = launch_prefill_scan<32>(sp, B, max_q_per_req, s); break;
    case 64: st = launch_prefill_scan<64>(sp, B, max_q_per_req, s); break;
    default: st = launch_prefill_scan<128>(sp, B, max_q_per_req, s); break;
  }
  if (st != QSA_OK) return st;
  // 2. per-token lengths and rows, own-block fix-up
  qsa::pre::PrepParams pp;
  pp.B = B;
  pp.n_tok = n_tokens;
  pp.cu_q = cu_q;
  pp.ctx_lens = ctx_lens;
  pp.q_idx = q_idx;
  pp.k_chunk = k_chunk;
  pp.d = cache->idx_dim;
  pp.max_blocks = max_blocks;
  pp.scores = scores;
  pp.tok_len = tok_len;
  pp.tok_row = tok_row;
  st = launch(true, qsa::pre::prefill_prep_kernel, dim3((unsigned)((n_tokens * 32LL + 255) / 256)),
              dim3(256), 0, s, pp);
  if (st != QSA_OK) return st;
  // 3. per-token selection over blocks 0 .. floor(p/4)
  qsa::topk::Params tp;
  tp.c = to_dev(cache);
  tp.B = n_tokens;
  tp.q_idx = q_idx;
  tp.ctx_lens = tok_len;
  tp.n_sel = nullptr;
  tp.max_blocks = max_blocks;
  tp.topk = topk;
  tp.sel = sel;
  tp.scores = scores;
  st = launch_select<qsa::topk::IntKeys>(tp, s);
  if (st != QSA_OK) return st;
  // 4. attention of every token over its kept tokens (one split: o, lse)
  return sparse_decode_call(cache, n_tokens, 1, Hq, q, q_dtype, tok_len, sel, topk, sm_scale, 1, 0,
                            1, o, lse, nullptr, nullptr, ws + lay.dec, lay.total - lay.dec, stream,
                            tok_row);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// qsa_index_topk_noalloc: qsa_index_topk for callers that cannot allocate.
//
// The score buffer of this variant is a fixed array in the library's device
// image: every GPU that loads libqsa.so holds kNoAllocScoreInts int32 (32 MiB)
// for it until the process exits.  Host code only ever sees a host-side
// stand-in for that array's name, so its device address is looked up once
// per device (cudaGetSymbolAddress, with that device current) and passed to
// the kernels.  Every call shares the array; the scan writes every score a
// selection then reads, so nothing in it needs clearing between calls, and
// calls that overlap on the GPU race on it.
// ---------------------------------------------------------------------------
namespace {

constexpr long long kNoAllocScoreInts = 8LL * 1024 * 1024;  // B * max_blocks limit
static __device__ __align__(256) int32_t g_noalloc_scores[kNoAllocScoreInts];

int32_t *g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the score array on the current device (set-up on first
// use per device); NULL if the runtime could not provide it.
int32_t *noalloc_scores_ptr() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mutex);
  if (!g_noalloc_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scores) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = static_cast<int32_t *>(ptr);
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" {

qsa_status qsa_index_topk_noalloc(const qsa_cache *cache, int32_t B, const int8_t *q_idx,
                                  const int32_t *ctx_lens, const int32_t *n_sel,
                                  int32_t max_blocks, int32_t topk, int32_t *sel,
                                  qsa_stream_t stream) {
  qsa_status st = check_cache(cache);
  if (st != QSA_OK) return st;
  if (B < 0) return QSA_ERR_INVALID_ARG;
  if (topk < 1 || topk > qsa::topk::kMaxTopk) return QSA_ERR_INVALID_ARG;
  if (max_blocks < 1 || max_blocks > (1 << 24)) return QSA_ERR_INVALID_ARG;
  if ((long long)B * max_blocks > kNoAllocScoreInts) return QSA_ERR_UNSUPPORTED;
  if (B == 0) return QSA_OK;
  if (!q_idx || !ctx_lens || !sel || !cache->kc) return QSA_ERR_INVALID_ARG;
  if (cache->idx_dim != 32 && cache->idx_dim != 64 && cache->idx_dim != 128)
    return QSA_ERR_UNSUPPORTED;
  if (!aligned(cache->kc, 16) || !aligned(q_idx, 4)) return QSA_ERR_INVALID_ARG;
  int32_t *scores = noalloc_scores_ptr();
  if (!scores) return QSA_ERR_CUDA;

  qsa::topk::Params p;
  p.c = to_dev(cache);
  p.B = B;
  p.q_idx = q_idx;
  p.ctx_lens = ctx_lens;
  p.n_sel = n_sel;
  p.max_blocks = max_blocks;
  p.topk = topk;
  p.sel = sel;
  p.scores = scores;
  return dispatch_index_topk(p, cache->idx_dim, cache->page_size,
                             reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
