// Host side of libnosa.so: argument validation, workspace layout, TMA
// descriptors and kernel launches for the C ABI declared in include/nosa.h.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "nosa.h"
#include "nosa_attn.cuh"
#include "nosa_attn_stop.cuh"
#include "nosa_common.cuh"
#include "nosa_kernels.cuh"
#include "nosa_select.cuh"

using namespace nosa;

namespace {

thread_local char g_err[512] = "";

nosa_status fail(nosa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

#define NOSA_CHECK(cond, ...) \
  do {                        \
    if (!(cond)) return fail(NOSA_EINVAL, __VA_ARGS__); \
  } while (0)

#define NOSA_CUDA(call)                                                                    \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess) return fail(NOSA_ECUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int n_groups(const nosa_config& c) { return c.B * c.Hkv; }
int max_sub(const nosa_config& c) { return c.max_blocks * (c.block_size / c.sub_block); }
int words(const nosa_config& c) { return (c.max_blocks + 31) / 32; }
int kk(const nosa_config& c) { return c.k_q + c.k_e; }

nosa_status check_cfg(const nosa_config* cp) {
  NOSA_CHECK(cp, "cfg is NULL");
  const nosa_config& c = *cp;
  NOSA_CHECK(c.B >= 1 && c.Hkv >= 1 && c.Hq >= c.Hkv && c.Hq % c.Hkv == 0,
             "bad heads: B=%d Hq=%d Hkv=%d", c.B, c.Hq, c.Hkv);
  const int G = c.Hq / c.Hkv;
  NOSA_CHECK(G == 1 || G == 2 || G == 4 || G == 8, "G = Hq/Hkv = %d not in {1,2,4,8}", G);
  NOSA_CHECK(c.d == 64 || c.d == 128, "d = %d not in {64,128}", c.d);
  NOSA_CHECK(c.block_size == 32 || c.block_size == 64 || c.block_size == 128,
             "block_size = %d not in {32,64,128}", c.block_size);
  NOSA_CHECK((c.sub_block == 8 || c.sub_block == 16 || c.sub_block == 32) &&
                 c.block_size % c.sub_block == 0,
             "sub_block = %d must be 8, 16 or 32 and divide block_size", c.sub_block);
  NOSA_CHECK(c.k_q >= 0 && c.k_e >= 0 && c.k_q + c.k_e >= 1, "bad budgets k_q=%d k_e=%d", c.k_q,
             c.k_e);
  NOSA_CHECK(c.max_blocks >= 1 && c.max_blocks <= kMaxBlocks, "max_blocks = %d not in [1, %d]",
             c.max_blocks, kMaxBlocks);
  NOSA_CHECK(kk(c) <= c.max_blocks, "k = %d > max_blocks = %d", kk(c), c.max_blocks);
  NOSA_CHECK(c.slots >= 1 && c.slots <= c.max_blocks, "slots = %d not in [1, max_blocks]", c.slots);
  NOSA_CHECK(c.n_score_rows == G || c.n_score_rows == 1, "n_score_rows = %d must be G or 1",
             c.n_score_rows);
  NOSA_CHECK(c.attn_split >= 0, "attn_split < 0");
  NOSA_CHECK(c.score_mode >= 0 && c.score_mode <= (NOSA_SCORE_WINDOW | NOSA_SCORE_SOFTMAX),
             "score_mode = %d: bits NOSA_SCORE_WINDOW | NOSA_SCORE_SOFTMAX only", c.score_mode);
  NOSA_CHECK(!(c.score_mode & NOSA_SCORE_SOFTMAX) || c.n_score_rows <= kMaxSoftRows,
             "softmax scoring supports at most %d scoring rows", kMaxSoftRows);
  NOSA_CHECK(c.stop_tau >= 0.f && c.stop_tau < 1e30f, "stop_tau must be >= 0 and finite");
  NOSA_CHECK(c.kc_bf16 == 0 || c.kc_bf16 == 1, "kc_bf16 must be 0 or 1");
  NOSA_CHECK(!(c.stop_tau > 0.f) || kk(c) <= kStopMaxK, "early stop supports k <= %d", kStopMaxK);
  NOSA_CHECK(c.scale > 0.f, "scale must be > 0");
  NOSA_CHECK(c.wait_us >= 0 && c.wait_us <= 60000000, "wait_us = %d not in [0, 60000000]", c.wait_us);
  const long long groups = (long long)c.B * c.Hkv;
  NOSA_CHECK(groups * c.slots * c.block_size < (1ll << 31), "too many pool rows for TMA coordinates");
  NOSA_CHECK(groups * kk(c) < (1ll << 31), "too many tasks");
  return NOSA_OK;
}

bool has_host(const nosa_state* st) { return st->host_k != nullptr; }

// Limit of the kernels' bounded waits, in ns.
unsigned long long wait_ns(const nosa_config& c) {
  return c.wait_us > 0 ? (unsigned long long)c.wait_us * 1000ull : kWaitLimitNs;
}

nosa_status check_state(const nosa_config& c, const nosa_state* st) {
  NOSA_CHECK(st, "state is NULL");
  const void* dev[] = {st->seq_len, st->kc, st->prev_sel, st->alive, st->last_used,
                       st->block_table, st->slot_owner, st->k_pool, st->v_pool, st->err};
  for (const void* p : dev) {
    NOSA_CHECK(p, "a device state buffer is NULL");
    NOSA_CHECK(aligned16(p), "state buffer %p not 16-byte aligned", p);
  }
  NOSA_CHECK((st->host_k == nullptr) == (st->host_v == nullptr), "host_k and host_v must both be set or both NULL");
  if (has_host(st)) {
    NOSA_CHECK(aligned16(st->host_k) && aligned16(st->host_v), "host pools not 16-byte aligned");
    NOSA_CHECK(c.slots >= kk(c) + 2, "offload needs slots >= k + 2 (slots=%d, k=%d)", c.slots, kk(c));
    for (const void* p : {(const void*)st->host_k, (const void*)st->host_v}) {
      cudaPointerAttributes at;
      cudaError_t e = cudaPointerGetAttributes(&at, p);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(NOSA_EINVAL, "host pool %p: %s", p, cudaGetErrorString(e));
      }
      NOSA_CHECK(at.type == cudaMemoryTypeHost && at.devicePointer == p,
                 "host pool %p is not pinned, device-mapped host memory", p);
    }
  } else {
    NOSA_CHECK(c.slots == c.max_blocks, "without host pools slots must equal max_blocks");
  }
  return NOSA_OK;
}

struct WsLayout {
  size_t scores, cnt_k1, cnt_attn, copy_list, copy_count, partials, ge_mask, sel_flag, copy_cnt,
      copy_flag, units, used, att_list, e_flag, total;
  int copy_stride;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const nosa_config& c) {
  WsLayout w;
  const size_t NG = n_groups(c);
  const int G = c.Hq / c.Hkv;
  w.copy_stride = (kk(c) + 1 > c.slots) ? kk(c) + 1 : c.slots;
  size_t off = 0;
  w.scores = off; off += up256(NG * c.max_blocks * 4);
  w.cnt_k1 = off; off += up256(NG * 4);
  w.cnt_attn = off; off += up256(NG * 4);
  w.copy_list = off; off += up256(NG * (size_t)w.copy_stride * 8);
  w.copy_count = off; off += up256(NG * 4);
  w.partials = off; off += up256(NG * kPartialSlots * (size_t)G * (c.d + 2) * 4);
  w.ge_mask = off; off += up256(NG * (size_t)words(c) * 4);
  w.sel_flag = off; off += up256(NG * kFlagStride * 4);
  w.copy_cnt = off; off += up256(NG * 4);
  w.copy_flag = off; off += up256(NG * kFlagStride * 4);
  // scoring variants: per-sub-block values (rows of logits for softmax, else one mean)
  const size_t urows = !c.score_mode ? 0 : ((c.score_mode & NOSA_SCORE_SOFTMAX) ? c.n_score_rows : 1);
  w.units = off; off += up256(NG * urows * (size_t)max_sub(c) * 4);
  w.used = off; off += up256((size_t)c.B * c.Hq * 4);
  w.att_list = off; off += up256(NG * (size_t)kk(c) * 4);
  w.e_flag = off; off += up256(NG * kFlagStride * 4);
  w.total = off;
  return w;
}

template <typename T>
T* ws_at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

nosa_status check_ws(const nosa_config& c, void* ws, size_t bytes) {
  NOSA_CHECK(ws && aligned16(ws), "workspace NULL or not 16-byte aligned");
  const size_t need = ws_layout(c).total;
  if (bytes < need) return fail(NOSA_ENOMEM, "workspace %zu bytes < %zu needed", bytes, need);
  return NOSA_OK;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

StepArgs step_args(const nosa_config& c, const nosa_state* st) {
  StepArgs a;
  memset(&a, 0, sizeof(a));
  a.kc = st->kc;
  a.kc16 = c.kc_bf16;
  a.seq_len = st->seq_len;
  a.max_blocks = c.max_blocks;
  a.max_sub = max_sub(c);
  a.bs = c.block_size;
  a.s = c.sub_block;
  a.slots = c.slots;
  a.scale = c.scale;
  a.total_pages = (long long)n_groups(c) * c.slots;
  a.k_pool = st->k_pool;
  a.v_pool = st->v_pool;
  a.host_k = st->host_k;
  a.host_v = st->host_v;
  a.block_table = st->block_table;
  a.prev_sel = st->prev_sel;
  a.alive = st->alive;
  a.k_q = c.k_q;
  a.k_e = c.k_e;
  a.slot_owner = st->slot_owner;
  a.last_used = st->last_used;
  a.err = st->err;
  a.wait_ns = wait_ns(c);
  return a;
}

void set_ws(StepArgs& a, const nosa_config& c, void* ws) {
  const WsLayout w = ws_layout(c);
  a.copy_list = ws_at<int2>(ws, w.copy_list);
  a.copy_stride = w.copy_stride;
  a.copy_count = ws_at<int32_t>(ws, w.copy_count);
  a.counters = ws_at<uint32_t>(ws, w.cnt_k1);
  a.ge_mask = ws_at<uint32_t>(ws, w.ge_mask);
  a.mode = c.score_mode;
  a.units = c.score_mode ? ws_at<float>(ws, w.units) : nullptr;
}

// ------------------------------------------------------------------ launches
// Score CTAs of 256 sub-blocks: about three waves on the Llama-shaped layer, each CTA short
// enough that an SM's CTAs finish at staggered times. (Larger chunks, one wave of about two CTAs
// per SM, streamed slower: fewer loads in flight.)
constexpr int kScoreChunk = 384;
// Shared-memory carveout (percent) of the score kernel, or -1 for the driver's choice, and the
// attention's shared memory for tile stages (its carveout is the largest shared split).
constexpr int kStepCarveout = -1;
constexpr int kAttnStageBudget = 110 * 1024;
// The fused step publishes each group's query-agnostic blocks ahead of the rest of its selection.
constexpr bool kEarlyGammaE = true;

// Sub-blocks per score CTA: the fewest chunks of at most kScoreChunk that cover max_sub, made
// equal (rounded up to kChunkAlign). max_sub is T/s plus one block's sub-blocks, so a fixed
// chunk would leave every group a last CTA of a few rows. Small batches take more, smaller
// chunks (down to kChunkAlign), so that the grid still fills the SMs about once.
int score_chunk_for(const nosa_config& c, int sms) {
  const int ms = max_sub(c);
  int C = (ms + kScoreChunk - 1) / kScoreChunk;
  const long long ng = n_groups(c);
  const int want = (int)((3LL * sms + ng - 1) / ng);  // three score CTAs per SM
  const int cmax = (ms + kChunkAlign - 1) / kChunkAlign;
  if (C < want) C = want < cmax ? want : cmax;
  const int even = (ms + C - 1) / C;
  return (even + kChunkAlign - 1) / kChunkAlign * kChunkAlign;
}

nosa_status score_chunk(const nosa_config& c, int* chunk) {
  int dev = 0, sms = 0;
  NOSA_CUDA(cudaGetDevice(&dev));
  NOSA_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  *chunk = score_chunk_for(c, sms);
  return NOSA_OK;
}

template <int D, bool FUSED, int VARIANT, bool KC16>
nosa_status launch_score_t(const nosa_config& c, const StepArgs& a0, cudaStream_t s) {
  StepArgs a = a0;
  nosa_status r = score_chunk(c, &a.chunk);
  if (r != NOSA_OK) return r;
  dim3 grid((max_sub(c) + a.chunk - 1) / a.chunk, n_groups(c));
  const size_t dsm = (FUSED ? score_su_offset(c.max_blocks) : 0) + (size_t)a.chunk * 4;
  auto k = score_kernel<D, FUSED, VARIANT, KC16>;
  if (dsm > 48 * 1024) NOSA_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm));
  if (kStepCarveout >= 0)
    NOSA_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, kStepCarveout));
  k<<<grid, kScoreThreads, dsm, s>>>(a);
  NOSA_CUDA(cudaGetLastError());
  return NOSA_OK;
}

template <int D, bool FUSED, int VARIANT>
nosa_status launch_score_kc(const nosa_config& c, const StepArgs& a, cudaStream_t s) {
  return c.kc_bf16 ? launch_score_t<D, FUSED, VARIANT, true>(c, a, s)
                   : launch_score_t<D, FUSED, VARIANT, false>(c, a, s);
}

template <bool FUSED>
nosa_status launch_score(const nosa_config& c, const StepArgs& a, cudaStream_t s) {
  if (FUSED && (c.score_mode & NOSA_SCORE_SOFTMAX))
    return c.d == 128 ? launch_score_kc<128, true, 2>(c, a, s) : launch_score_kc<64, true, 2>(c, a, s);
  if (FUSED && c.score_mode)
    return c.d == 128 ? launch_score_kc<128, true, 1>(c, a, s) : launch_score_kc<64, true, 1>(c, a, s);
  return c.d == 128 ? launch_score_kc<128, FUSED, 0>(c, a, s) : launch_score_kc<64, FUSED, 0>(c, a, s);
}

nosa_status launch_sel_kernel(void (*k)(StepArgs), const nosa_config& c, const StepArgs& a,
                              cudaStream_t s) {
  const size_t dsm = sel_smem_bytes(c.max_blocks);
  if (dsm > 48 * 1024)
    NOSA_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm));
  k<<<n_groups(c), kSelThreads, dsm, s>>>(a);
  NOSA_CUDA(cudaGetLastError());
  return NOSA_OK;
}

// CTAs of the flag-driven copy: 64 x 256 threads x 128 bytes in flight is about 2 MiB, well
// above what PCIe needs to stay busy, while leaving the SMs to the score and attention CTAs.
constexpr int kCopyCtas = 64;

nosa_status launch_copy(const nosa_config& c, const nosa_state* st, void* ws, cudaStream_t s,
                        bool flags = false) {
  const WsLayout w = ws_layout(c);
  CopyArgs ca;
  ca.copy_list = ws_at<int2>(ws, w.copy_list);
  ca.copy_stride = w.copy_stride;
  ca.copy_count = ws_at<int32_t>(ws, w.copy_count);
  ca.host_k = reinterpret_cast<const uint4*>(st->host_k);
  ca.host_v = reinterpret_cast<const uint4*>(st->host_v);
  ca.k_pool = reinterpret_cast<uint4*>(st->k_pool);
  ca.v_pool = reinterpret_cast<uint4*>(st->v_pool);
  ca.max_blocks = c.max_blocks;
  ca.page_vec = c.block_size * c.d * 2 / 16;
  ca.sel_flag = flags ? ws_at<uint32_t>(ws, w.sel_flag) : nullptr;
  ca.copy_cnt = ws_at<uint32_t>(ws, w.copy_cnt);
  ca.copy_flag = ws_at<uint32_t>(ws, w.copy_flag);
  ca.err = st->err;
  ca.wait_ns = wait_ns(c);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(n_groups(c), 8);
  lc.blockDim = dim3(256);
  lc.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  if (flags) {
    lc.gridDim = dim3(kCopyCtas);
    NOSA_CUDA(cudaLaunchKernelEx(&lc, copy_seq_kernel, ca, (int)n_groups(c)));
  } else {
    NOSA_CUDA(cudaLaunchKernelEx(&lc, copy_kernel, ca));
  }
  return NOSA_OK;
}

// ---- TMA descriptors (driver entry point fetched through the runtime; no -lcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

nosa_status get_encode(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  if (!cached) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    NOSA_CUDA(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !p) return fail(NOSA_ECUDA, "cuTensorMapEncodeTiled unavailable");
    cached = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = cached;
  return NOSA_OK;
}

nosa_status make_pool_map(CUtensorMap* m, const nosa_config& c, void* pool) {
  EncodeTiledFn enc;
  nosa_status r = get_encode(&enc);
  if (r != NOSA_OK) return r;
  const cuuint64_t rows = (cuuint64_t)n_groups(c) * c.slots * c.block_size;
  cuuint64_t dims[2] = {(cuuint64_t)c.d, rows};
  cuuint64_t strides[1] = {(cuuint64_t)c.d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)c.block_size};
  cuuint32_t estr[2] = {1, 1};
  CUresult e = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (e != CUDA_SUCCESS) return fail(NOSA_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)e);
  return NOSA_OK;
}

// Tasks ((group, block) pairs) per attention CTA. split > 0: the caller's width; finest: the
// smallest width the partial slots allow; otherwise the automatic rule below. target = the
// resident attention CTAs (SMs x CTAs per SM), stage = bytes of one block's K and V pages.
int attn_split_for(int split, int k, int total, long long target, int sms, int stage, bool finest) {
  const int wmin = (k + kPartialSlots - 2) / (kPartialSlots - 1);
  int W = split;
  if (W <= 0 && finest) W = wmin;
  if (W <= 0) {
    // Prefer a divisor of k: every CTA then holds one segment of one group and never flushes
    // in mid-stream. Aim at about one CTA per resident slot: a single wave pays each CTA's
    // start (flag, selection, first tiles) and flush once per slot (Llama-shaped layer:
    // W = 32 gives 55 us of attention against 58 us at W = 16, and a shorter step).
    const double want = (double)total / (double)target;
    int best = 0;
    double best_d = 1e30;
    for (int d = wmin; d <= k; ++d) {
      if (k % d) continue;
      const double dist = d > want ? d / want : want / d;
      if (dist < best_d) { best_d = dist; best = d; }
    }
    W = (best > 0 && best_d <= 2.0) ? best : (int)((total + target - 1) / target);
    // Few selected pages per group (at most 512 KB of K and V), groups enough to spread over
    // the SMs and few enough for one wave: one CTA per group. Each group's attention then
    // starts as soon as its selection is published and needs no merge across CTAs (sweep,
    // T=65536, bs=64, 1 %: 51 us per step against 61 us with W = 3).
    const long long ng = total / k;
    if (ng <= target && 4 * ng >= sms && (long long)k * stage <= 512 * 1024) W = k;
  }
  if (W < wmin) W = wmin;
  if (W < 1) W = 1;
  return W;
}

// finest: the smallest split width the partial slots allow (used when the attention of each
// group waits for that group's page copies: groups become ready one after another over the
// whole PCIe transfer, so spreading each group over more CTAs shortens the last group's tail).
template <int D, int BS>
nosa_status launch_attn_t(const nosa_config& c, AttnArgs a, const CUtensorMap& tk, const CUtensorMap& tv,
                          cudaStream_t s, bool finest, bool pdl = true) {
  using SH = AttnShape<D, BS>;
  int stages = kAttnStageBudget / SH::STAGE;
  stages = stages < 2 ? 2 : (stages > kMaxStages ? kMaxStages : stages);
  const size_t smem = SH::smem_bytes(stages);
  auto k = attn_kernel<D, BS>;
  NOSA_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  NOSA_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared));
  int dev = 0, sms = 0, per_sm = 0;
  NOSA_CUDA(cudaGetDevice(&dev));
  NOSA_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  NOSA_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, SH::THREADS, smem));
  if (per_sm < 1) per_sm = 1;
  const long long target = (long long)sms * per_sm;
  const int W = attn_split_for(c.attn_split, a.k, a.total, target, sms, SH::STAGE, finest);
  a.W = W;
  a.stages = stages;
  const int grid = (a.total + W - 1) / W;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(grid);
  lc.blockDim = dim3(SH::THREADS);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = pdl ? 1 : 0;
  NOSA_CUDA(cudaLaunchKernelEx(&lc, k, tk, tv, a));
  return NOSA_OK;
}

template <int D, int BS>
nosa_status launch_attn_stop_t(const nosa_config& c, AttnArgs a, StopArgs x, const CUtensorMap& tk,
                               const CUtensorMap& tv, cudaStream_t s, bool pdl) {
  using SH = AttnShape<D, BS>;
  using SS = StopShape<D, BS>;
  // one CTA per group, one per SM: spend the shared memory on stages
  const int G = c.Hq / c.Hkv;
  int stages = (int)((227 * 1024 - 1024 - SS::extra_bytes(G)) / SH::STAGE);
  stages = stages < 2 ? 2 : (stages > kMaxStages ? kMaxStages : stages);
  const size_t smem = SS::smem_bytes(stages, G);
  auto k = attn_stop_kernel<D, BS>;
  NOSA_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  a.stages = stages;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(n_groups(c));
  lc.blockDim = dim3(SH::THREADS);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = pdl ? 1 : 0;
  NOSA_CUDA(cudaLaunchKernelEx(&lc, k, tk, tv, a, x));
  return NOSA_OK;
}

// Arguments of the split-K attention over the state's pools. partials / counters: the
// scratch of the split-K merge (the workspace's, or the no-allocation entry point's).
AttnArgs attn_args(const nosa_config& c, const nosa_state* st, const uint16_t* q, const int32_t* sel,
                   float* out, float* partials, uint32_t* counters) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q;
  a.sel = sel;
  a.seq_len = st->seq_len;
  a.block_table = st->block_table;
  a.out = out;
  a.partials = partials;
  a.counters = counters;
  a.err = st->err;
  a.Hq = c.Hq;
  a.Hkv = c.Hkv;
  a.G = c.Hq / c.Hkv;
  a.k = kk(c);
  a.max_blocks = c.max_blocks;
  a.total = n_groups(c) * kk(c);
  a.total_pages = (long long)n_groups(c) * c.slots;
  a.scale_log2 = c.scale * 1.4426950408889634f;
  a.identity = !has_host(st);
  a.wait_ns = wait_ns(c);
  return a;
}

nosa_status make_pool_maps(const nosa_config& c, const nosa_state* st, CUtensorMap* tk, CUtensorMap* tv) {
  nosa_status r = make_pool_map(tk, c, st->k_pool);
  if (r != NOSA_OK) return r;
  return make_pool_map(tv, c, st->v_pool);
}

// The split-K attention kernel instantiated for the configuration's head dim and block size.
nosa_status dispatch_attn(const nosa_config& c, const AttnArgs& a, const CUtensorMap& tk,
                          const CUtensorMap& tv, cudaStream_t s, bool finest, bool pdl) {
  if (c.d == 128) {
    if (c.block_size == 32) return launch_attn_t<128, 32>(c, a, tk, tv, s, finest, pdl);
    if (c.block_size == 64) return launch_attn_t<128, 64>(c, a, tk, tv, s, finest, pdl);
    return launch_attn_t<128, 128>(c, a, tk, tv, s, finest, pdl);
  }
  if (c.block_size == 32) return launch_attn_t<64, 32>(c, a, tk, tv, s, finest, pdl);
  if (c.block_size == 64) return launch_attn_t<64, 64>(c, a, tk, tv, s, finest, pdl);
  return launch_attn_t<64, 128>(c, a, tk, tv, s, finest, pdl);
}

// ready: per-group flags the attention waits on (and clears), or NULL to wait for the
// previous grid as a whole. pdl: may start while the previous kernel on the stream runs.
// early: the score kernel of the same step publishes each group's query-agnostic blocks
// ahead of the rest of its selection (per-group flags only).
nosa_status launch_attn(const nosa_config& c, const nosa_state* st, const uint16_t* q, const int32_t* sel,
                        float* out, void* ws, cudaStream_t s, uint32_t* ready = nullptr,
                        bool pdl = true, bool early = false) {
  CUtensorMap tk, tv;
  nosa_status r = make_pool_maps(c, st, &tk, &tv);
  if (r != NOSA_OK) return r;
  const WsLayout w = ws_layout(c);
  AttnArgs a = attn_args(c, st, q, sel, out, ws_at<float>(ws, w.partials), ws_at<uint32_t>(ws, w.cnt_attn));
  a.sel_flag = ready;
  if (early && ready) {
    a.att_list = ws_at<int32_t>(ws, w.att_list);
    a.e_flag = ws_at<uint32_t>(ws, w.e_flag);
  }
  if (c.stop_tau > 0.f) {
    // early stop: one CTA per group, each waiting for its own group's flag (or the whole grid)
    StopArgs x;
    x.scores = ws_at<float>(ws, w.scores);
    x.tau = c.stop_tau;
    x.used = ws_at<int32_t>(ws, w.used);
    if (c.d == 128) {
      if (c.block_size == 32) return launch_attn_stop_t<128, 32>(c, a, x, tk, tv, s, pdl);
      if (c.block_size == 64) return launch_attn_stop_t<128, 64>(c, a, x, tk, tv, s, pdl);
      return launch_attn_stop_t<128, 128>(c, a, x, tk, tv, s, pdl);
    }
    if (c.block_size == 32) return launch_attn_stop_t<64, 32>(c, a, x, tk, tv, s, pdl);
    if (c.block_size == 64) return launch_attn_stop_t<64, 64>(c, a, x, tk, tv, s, pdl);
    return launch_attn_stop_t<64, 128>(c, a, x, tk, tv, s, pdl);
  }
  const bool finest = ready != nullptr && has_host(st);
  return dispatch_attn(c, a, tk, tv, s, finest, pdl);
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* nosa_status_string(nosa_status s) {
  switch (s) {
    case NOSA_OK: return "ok";
    case NOSA_EINVAL: return "invalid argument";
    case NOSA_ENOMEM: return "workspace too small";
    case NOSA_ECUDA: return "CUDA runtime error";
    case NOSA_EDEVICE: return "device-side fault recorded";
    case NOSA_ETIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* nosa_last_error(void) { return g_err; }

nosa_status nosa_state_sizes(const nosa_config* cfg, nosa_sizes* out) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  NOSA_CHECK(out, "out is NULL");
  const nosa_config& c = *cfg;
  const size_t NG = n_groups(c);
  out->seq_len = NG * 4;
  out->kc = NG * max_sub(c) * (size_t)c.d * (c.kc_bf16 ? 2 : 4);
  out->prev_sel = NG * words(c) * 4;
  out->alive = NG * words(c) * 4;
  out->last_used = NG * c.max_blocks * 4;
  out->block_table = NG * c.max_blocks * 4;
  out->slot_owner = NG * c.slots * 4;
  out->k_pool = NG * c.slots * (size_t)c.block_size * c.d * 2;
  out->v_pool = out->k_pool;
  out->host_k = NG * c.max_blocks * (size_t)c.block_size * c.d * 2;
  out->host_v = out->host_k;
  out->err = 4;
  return NOSA_OK;
}

nosa_status nosa_workspace_size(const nosa_config* cfg, size_t* bytes) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  NOSA_CHECK(bytes, "bytes is NULL");
  *bytes = ws_layout(*cfg).total;
  return NOSA_OK;
}

nosa_status nosa_workspace_init(void* ws, size_t bytes, void* stream) {
  NOSA_CHECK(ws && aligned16(ws), "workspace NULL or not 16-byte aligned");
  NOSA_CUDA(cudaMemsetAsync(ws, 0, bytes, as_stream(stream)));
  return NOSA_OK;
}

nosa_status nosa_state_init(const nosa_config* cfg, const nosa_state* st, const int32_t* prefill_len,
                            const uint8_t* resident, void* ws, size_t ws_bytes, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  if ((r = check_ws(c, ws, ws_bytes)) != NOSA_OK) return r;
  NOSA_CHECK(prefill_len, "prefill_len is NULL");
  cudaStream_t s = as_stream(stream);
  NOSA_CUDA(cudaMemsetAsync(st->err, 0, 4, s));
  const WsLayout w = ws_layout(c);
  InitArgs a;
  a.prefill_len = prefill_len;
  a.resident = resident;
  a.seq_len = st->seq_len;
  a.prev_sel = st->prev_sel;
  a.alive = st->alive;
  a.last_used = st->last_used;
  a.block_table = st->block_table;
  a.slot_owner = st->slot_owner;
  a.copy_list = ws_at<int2>(ws, w.copy_list);
  a.copy_stride = w.copy_stride;
  a.copy_count = ws_at<int32_t>(ws, w.copy_count);
  a.err = st->err;
  a.Hkv = c.Hkv;
  a.bs = c.block_size;
  a.max_blocks = c.max_blocks;
  a.slots = c.slots;
  a.host = has_host(st) ? 1 : 0;
  init_tables_kernel<<<n_groups(c), 256, 0, s>>>(a);
  NOSA_CUDA(cudaGetLastError());
  const uint16_t* src = has_host(st) ? st->host_k : st->k_pool;
  const int ppg = has_host(st) ? c.max_blocks : c.slots;
  const int subs = 256 / c.d * 4;
  dim3 g((max_sub(c) + subs - 1) / subs, n_groups(c));
  if (c.d == 128)
    if (c.kc_bf16) init_kc_kernel<128, true><<<g, 256, 0, s>>>(prefill_len, c.Hkv, src, ppg, st->kc, max_sub(c), c.block_size, c.sub_block);
    else init_kc_kernel<128, false><<<g, 256, 0, s>>>(prefill_len, c.Hkv, src, ppg, st->kc, max_sub(c), c.block_size, c.sub_block);
  else
    if (c.kc_bf16) init_kc_kernel<64, true><<<g, 256, 0, s>>>(prefill_len, c.Hkv, src, ppg, st->kc, max_sub(c), c.block_size, c.sub_block);
    else init_kc_kernel<64, false><<<g, 256, 0, s>>>(prefill_len, c.Hkv, src, ppg, st->kc, max_sub(c), c.block_size, c.sub_block);
  NOSA_CUDA(cudaGetLastError());
  if (has_host(st)) return launch_copy(c, st, ws, s);
  return NOSA_OK;
}

nosa_status nosa_append(const nosa_config* cfg, const nosa_state* st, const uint16_t* k_new,
                        const uint16_t* v_new, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  NOSA_CHECK(k_new && v_new && aligned16(k_new) && aligned16(v_new), "k_new/v_new NULL or misaligned");
  StepArgs a = step_args(c, st);
  a.k_new = k_new;
  a.v_new = v_new;
  if (c.d == 128) append_kernel<128><<<n_groups(c), 128, 0, as_stream(stream)>>>(a);
  else append_kernel<64><<<n_groups(c), 128, 0, as_stream(stream)>>>(a);
  NOSA_CUDA(cudaGetLastError());
  return NOSA_OK;
}

nosa_status nosa_score_blocks(const nosa_config* cfg, const nosa_state* st, const uint16_t* rows,
                              float* block_scores, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  NOSA_CHECK(rows && block_scores && aligned16(rows) && aligned16(block_scores),
             "score rows / block_scores NULL or misaligned");
  NOSA_CHECK(c.score_mode == 0, "scoring variants need the whole group's values before any block "
                                "score: use nosa_step or nosa_plan_ahead");
  StepArgs a = step_args(c, st);
  a.rows = rows;
  a.R = c.n_score_rows;
  a.block_scores = block_scores;
  return launch_score<false>(c, a, as_stream(stream));
}

nosa_status nosa_select(const nosa_config* cfg, const nosa_state* st, const float* block_scores,
                        const float* evict, int32_t* sel, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  NOSA_CHECK(block_scores && evict && sel && aligned16(block_scores) && aligned16(evict) && aligned16(sel),
             "select buffers NULL or misaligned");
  StepArgs a = step_args(c, st);
  a.block_scores = const_cast<float*>(block_scores);
  a.evict = evict;
  a.sel = sel;
  return launch_sel_kernel(select_kernel, c, a, as_stream(stream));
}

nosa_status nosa_gather(const nosa_config* cfg, const nosa_state* st, const int32_t* sel,
                        int32_t* miss_count, void* ws, size_t ws_bytes, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  if ((r = check_ws(c, ws, ws_bytes)) != NOSA_OK) return r;
  NOSA_CHECK(sel && miss_count && aligned16(sel) && aligned16(miss_count), "sel/miss_count NULL or misaligned");
  cudaStream_t s = as_stream(stream);
  if (!has_host(st)) {
    NOSA_CUDA(cudaMemsetAsync(miss_count, 0, (size_t)n_groups(c) * 4, s));
    return NOSA_OK;
  }
  StepArgs a = step_args(c, st);
  set_ws(a, c, ws);
  a.sel = const_cast<int32_t*>(sel);
  a.miss_count = miss_count;
  if ((r = launch_sel_kernel(plan_kernel, c, a, s)) != NOSA_OK) return r;
  return launch_copy(c, st, ws, s);
}

nosa_status nosa_decode_attn(const nosa_config* cfg, const nosa_state* st, const uint16_t* q,
                             const int32_t* sel, float* out, void* ws, size_t ws_bytes, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  if ((r = check_ws(c, ws, ws_bytes)) != NOSA_OK) return r;
  NOSA_CHECK(q && sel && out && aligned16(q) && aligned16(sel) && aligned16(out), "q/sel/out NULL or misaligned");
  NOSA_CHECK(!(c.stop_tau > 0.f), "early stop visits blocks by the step's scores: use nosa_step");
  return launch_attn(c, st, q, sel, out, ws, as_stream(stream));
}

nosa_status nosa_step(const nosa_config* cfg, const nosa_state* st, const uint16_t* q,
                      const uint16_t* score_rows, const uint16_t* k_new, const uint16_t* v_new,
                      const float* evict, int32_t* sel, float* out, int32_t* miss_count, void* ws,
                      size_t ws_bytes, void* stream, void* const* events) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  if ((r = check_ws(c, ws, ws_bytes)) != NOSA_OK) return r;
  NOSA_CHECK(q && k_new && v_new && evict && sel && out && miss_count, "step buffer is NULL");
  const void* ptrs[] = {q, k_new, v_new, evict, sel, out, miss_count};
  for (const void* p : ptrs) NOSA_CHECK(aligned16(p), "step buffer %p not 16-byte aligned", p);
  NOSA_CHECK(score_rows || c.n_score_rows == c.Hq / c.Hkv, "score_rows NULL requires n_score_rows == G");
  NOSA_CHECK(!score_rows || aligned16(score_rows), "score_rows misaligned");
  cudaStream_t s = as_stream(stream);
  auto rec = [&](int i) -> nosa_status {
    if (events && events[i]) NOSA_CUDA(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s));
    return NOSA_OK;
  };
  if ((r = rec(0)) != NOSA_OK) return r;
  StepArgs a = step_args(c, st);
  set_ws(a, c, ws);
  a.rows = score_rows ? score_rows : q;
  a.R = c.n_score_rows;
  a.block_scores = ws_at<float>(ws, ws_layout(c).scores);
  a.k_new = k_new;
  a.v_new = v_new;
  a.evict = evict;
  a.sel = sel;
  a.miss_count = miss_count;
  a.append = 1;
  // Per-group flags chain the kernels group by group: the attention of a group starts as soon
  // as that group's selection is published or, with host pools, as soon as its page copies
  // (which themselves start on the group's published plan) have landed. With events each
  // kernel waits for the previous one as a whole, so that the events time kernels alone.
  const WsLayout w = ws_layout(c);
  const bool flags = !events;
  // early stop ranks the whole selection before its first block: no early Gamma_e there
  const bool early = flags && kEarlyGammaE && !(c.stop_tau > 0.f);
  a.sel_flag = flags ? ws_at<uint32_t>(ws, w.sel_flag) : nullptr;
  if (early) {
    // the query-agnostic blocks of a group are attended as soon as they are chosen
    a.att_list = ws_at<int32_t>(ws, w.att_list);
    a.e_flag = ws_at<uint32_t>(ws, w.e_flag);
  }
  uint32_t* ready = !flags ? nullptr
                           : ws_at<uint32_t>(ws, has_host(st) ? w.copy_flag : w.sel_flag);
  if ((r = launch_score<true>(c, a, s)) != NOSA_OK) return r;
  if ((r = rec(1)) != NOSA_OK) return r;
  if (has_host(st) && (r = launch_copy(c, st, ws, s, flags)) != NOSA_OK) return r;
  if ((r = rec(2)) != NOSA_OK) return r;
  if ((r = launch_attn(c, st, q, sel, out, ws, s, ready, true, early)) != NOSA_OK) return r;
  return rec(3);
}

nosa_status nosa_step_geometry(const nosa_config* cfg, int32_t host_pools, int32_t sms,
                               int32_t attn_ctas_per_sm, nosa_geometry* out) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  NOSA_CHECK(out, "out is NULL");
  NOSA_CHECK(sms >= 1 && attn_ctas_per_sm >= 1, "sms (%d) and attn_ctas_per_sm (%d) must be >= 1", sms,
             attn_ctas_per_sm);
  const nosa_config& c = *cfg;
  const int chunk = score_chunk_for(c, sms);
  out->score_chunk = chunk;
  out->score_ctas = n_groups(c) * ((max_sub(c) + chunk - 1) / chunk);
  const int k = kk(c), total = n_groups(c) * k;
  if (c.stop_tau > 0.f) {
    // early stop: one CTA per group visits its blocks in order
    out->attn_tasks_per_cta = k;
    out->attn_ctas = n_groups(c);
    return NOSA_OK;
  }
  // K and V pages of one block: 2 x bs x d bf16 values
  const int W = attn_split_for(c.attn_split, k, total, (long long)sms * attn_ctas_per_sm, sms,
                               4 * c.block_size * c.d, host_pools != 0);
  out->attn_tasks_per_cta = W;
  out->attn_ctas = (total + W - 1) / W;
  return NOSA_OK;
}

nosa_status nosa_step_launches(const nosa_config* cfg, const nosa_state* st, int32_t* kernels) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  NOSA_CHECK(kernels, "kernels is NULL");
  *kernels = has_host(st) ? 3 : 2;  // score + selection, [page copies,] attention
  return NOSA_OK;
}

nosa_status nosa_plan_ahead(const nosa_config* cfg, const nosa_state* st, const uint16_t* score_rows,
                            const float* evict, int32_t* sel, int32_t* miss_count, void* ws,
                            size_t ws_bytes, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  if ((r = check_ws(c, ws, ws_bytes)) != NOSA_OK) return r;
  NOSA_CHECK(score_rows && evict && sel && miss_count, "plan_ahead buffer is NULL");
  NOSA_CHECK(!(c.stop_tau > 0.f), "early stop is defined on the standard step order (nosa_step)");
  const void* ptrs[] = {score_rows, evict, sel, miss_count};
  for (const void* p : ptrs) NOSA_CHECK(aligned16(p), "plan_ahead buffer %p not 16-byte aligned", p);
  cudaStream_t s = as_stream(stream);
  const WsLayout w = ws_layout(c);
  StepArgs a = step_args(c, st);
  set_ws(a, c, ws);
  a.rows = score_rows;
  a.R = c.n_score_rows;
  a.block_scores = ws_at<float>(ws, w.scores);
  a.evict = evict;
  a.sel = sel;
  a.miss_count = miss_count;
  a.append = 0;
  a.sel_flag = ws_at<uint32_t>(ws, w.sel_flag);
  return launch_score<true>(c, a, s);
}

nosa_status nosa_prefetch(const nosa_config* cfg, const nosa_state* st, void* ws, size_t ws_bytes,
                          void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  if ((r = check_ws(c, ws, ws_bytes)) != NOSA_OK) return r;
  if (!has_host(st)) return NOSA_OK;
  return launch_copy(c, st, ws, as_stream(stream), true);
}

nosa_status nosa_attend(const nosa_config* cfg, const nosa_state* st, const uint16_t* q,
                        const uint16_t* k_new, const uint16_t* v_new, const int32_t* sel, float* out,
                        void* ws, size_t ws_bytes, void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  if ((r = check_ws(c, ws, ws_bytes)) != NOSA_OK) return r;
  NOSA_CHECK(q && k_new && v_new && sel && out, "attend buffer is NULL");
  NOSA_CHECK(!(c.stop_tau > 0.f), "early stop is defined on the standard step order (nosa_step)");
  const void* ptrs[] = {q, k_new, v_new, sel, out};
  for (const void* p : ptrs) NOSA_CHECK(aligned16(p), "attend buffer %p not 16-byte aligned", p);
  cudaStream_t s = as_stream(stream);
  const WsLayout w = ws_layout(c);
  uint32_t* ready = ws_at<uint32_t>(ws, has_host(st) ? w.copy_flag : w.sel_flag);
  StepArgs a = step_args(c, st);
  a.k_new = k_new;
  a.v_new = v_new;
  a.ready = ready;
  if (c.d == 128) append_kernel<128><<<n_groups(c), 128, 0, s>>>(a);
  else append_kernel<64><<<n_groups(c), 128, 0, s>>>(a);
  NOSA_CUDA(cudaGetLastError());
  // no programmatic early start: the attention reads the length the append just wrote
  return launch_attn(c, st, q, sel, out, ws, s, ready, false);
}

nosa_status nosa_stop_counts(const nosa_config* cfg, const void* ws, size_t ws_bytes, int32_t* used,
                             void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_ws(c, const_cast<void*>(ws), ws_bytes)) != NOSA_OK) return r;
  NOSA_CHECK(used && aligned16(used), "used NULL or misaligned");
  NOSA_CUDA(cudaMemcpyAsync(used, static_cast<const uint8_t*>(ws) + ws_layout(c).used,
                            (size_t)c.B * c.Hq * 4, cudaMemcpyDeviceToDevice, as_stream(stream)));
  return NOSA_OK;
}

nosa_status nosa_check_device(const nosa_state* st, void* stream, uint32_t* err_out) {
  NOSA_CHECK(st && st->err, "state/err is NULL");
  uint32_t e = 0;
  NOSA_CUDA(cudaMemcpyAsync(&e, st->err, 4, cudaMemcpyDeviceToHost, as_stream(stream)));
  NOSA_CUDA(cudaStreamSynchronize(as_stream(stream)));
  if (err_out) *err_out = e;
  if (e & NOSA_ERR_TIMEOUT) return fail(NOSA_ETIMEOUT, "device wait timed out (err=0x%x)", e);
  if (e) return fail(NOSA_EDEVICE, "device fault bits 0x%x", e);
  return NOSA_OK;
}

}  // extern "C"

// ====================================================================== no-allocation attention
// nosa_decode_attn_noalloc: the split-K attention of nosa_decode_attn with its scratch (the
// per-group online-softmax partials and the last-arriver counters) placed in the array below
// instead of the caller's workspace. The array lives in this library's device image, so every
// GPU that loads the library holds it until the process exits.
#include <mutex>

namespace {
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code the array's name
// is only a host-side stand-in, so the address is looked up once per device (with that device
// current) and cached.
nosa_status noalloc_scratch(void** out) {
  int dev = 0;
  NOSA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(NOSA_EINVAL, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(NOSA_ECUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return NOSA_OK;
}
}  // namespace

extern "C" nosa_status nosa_decode_attn_noalloc(const nosa_config* cfg, const nosa_state* st,
                                                const uint16_t* q, const int32_t* sel, float* out,
                                                void* stream) {
  nosa_status r = check_cfg(cfg);
  if (r != NOSA_OK) return r;
  const nosa_config& c = *cfg;
  if ((r = check_state(c, st)) != NOSA_OK) return r;
  NOSA_CHECK(q && sel && out && aligned16(q) && aligned16(sel) && aligned16(out),
             "q/sel/out NULL or misaligned");
  NOSA_CHECK(!(c.stop_tau > 0.f), "early stop visits blocks by the step's scores: use nosa_step");
  const size_t NG = n_groups(c);
  const size_t part_bytes = up256(NG * kPartialSlots * (size_t)(c.Hq / c.Hkv) * (c.d + 2) * 4);
  const size_t need = part_bytes + up256(NG * 4);
  if (need > kNoAllocScratchBytes)
    return fail(NOSA_ENOMEM, "nosa_decode_attn_noalloc needs %zu bytes of static scratch; the limit is %zu "
                "(use nosa_decode_attn with a workspace)", need, kNoAllocScratchBytes);
  void* base = nullptr;
  if ((r = noalloc_scratch(&base)) != NOSA_OK) return r;
  cudaStream_t s = as_stream(stream);
  // every check (the tensor maps included) before the first work is queued on the stream
  CUtensorMap tk, tv;
  if ((r = make_pool_maps(c, st, &tk, &tv)) != NOSA_OK) return r;
  uint32_t* counters = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(base) + part_bytes);
  // the array keeps the previous call's contents: the last-arriver counters must start at zero
  NOSA_CUDA(cudaMemsetAsync(counters, 0, NG * 4, s));
  const AttnArgs a = attn_args(c, st, q, sel, out, static_cast<float*>(base), counters);
  return dispatch_attn(c, a, tk, tv, s, /*finest=*/false, /*pdl=*/true);
}

// ====================================================================== PCIe read ceiling
// nosa_uva_read_probe: host -> device copy by 16-byte loads over UVA, four loads in flight
// per thread, grid-stride. The gather kernel reads host pages the same way, so the probe's
// rate is the ceiling the gather's achieved PCIe bandwidth is reported against.
namespace {
__global__ void __launch_bounds__(256) uva_read_kernel(const uint4* __restrict__ src,
                                                       uint4* __restrict__ dst, size_t n) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n; i += 4 * stride) {
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) r[u] = src[i + u * stride];
#pragma unroll
    for (int u = 0; u < 4; ++u) dst[i + u * stride] = r[u];
  }
  for (; i < n; i += stride) dst[i] = src[i];
}
}  // namespace

extern "C" nosa_status nosa_uva_read_probe(const void* host, void* dev, size_t bytes, int ctas,
                                           void* stream) {
  NOSA_CHECK(host && dev, "host/dev is NULL");
  NOSA_CHECK(aligned16(host) && aligned16(dev) && bytes % 16 == 0,
             "host, dev and bytes must be multiples of 16");
  NOSA_CHECK(ctas >= 0, "ctas < 0");
  cudaPointerAttributes at;
  cudaError_t e = cudaPointerGetAttributes(&at, host);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(NOSA_EINVAL, "host %p: %s", host, cudaGetErrorString(e));
  }
  NOSA_CHECK(at.type == cudaMemoryTypeHost && at.devicePointer == host,
             "host %p is not pinned, device-mapped host memory", host);
  if (bytes == 0) return NOSA_OK;
  if (ctas == 0) {
    int d = 0, sms = 0;
    NOSA_CUDA(cudaGetDevice(&d));
    NOSA_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d));
    ctas = 4 * sms;
  }
  uva_read_kernel<<<ctas, 256, 0, as_stream(stream)>>>(static_cast<const uint4*>(host),
                                                       static_cast<uint4*>(dev), bytes / 16);
  NOSA_CUDA(cudaGetLastError());
  return NOSA_OK;
}
