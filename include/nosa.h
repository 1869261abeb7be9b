/*
 * nosa.h -- C ABI of libnosa.so: one decode step of NOSA block-sparse attention
 * over an offloadable, paged KV cache, on one B200 (sm_100a).
 *
 * Method: NOSA, "Native and Offloadable Sparse Attention" (technical summary,
 * gist.science/es/paper/2510.13602, section "Metodologia" 1 and 2; blog
 * summary at blogs.edgentiq.com). Per GQA group (b, g): two-stage pooled block
 * scores, the union of a query-aware top-k_q and a query-agnostic top-k_e
 * eviction set (a block left out of the latter never returns to it), a paged
 * gather whose misses are read from pinned host memory over UVA, and split-K
 * flash-decoding with an online-softmax combine. SparDA ("Sparse Decoupled
 * Attention", gist.science/de/paper/2606.04511, section 2, "Kompakter
 * Forecast-Indexer") supplies the one-forecast-row scoring variant.
 *
 * Conventions (every entry point):
 *  - Returns nosa_status; never aborts, throws or prints. A call refused for its
 *    arguments (NOSA_EINVAL, NOSA_ENOMEM) launches nothing: every check comes
 *    before the first launch. NOSA_ECUDA reports a CUDA error, which may come
 *    after some of the call's kernels were launched. nosa_last_error() gives a
 *    one-line reason (thread-local).
 *  - Runs on the calling thread's current device: pointers and the stream must
 *    belong to it (the library reads that device's SM count and sets its kernel
 *    attributes there).
 *  - Calls on different states and workspaces may run concurrently on any
 *    streams. Calls that share a state or a workspace must be ordered (one
 *    stream, or events): the kernels keep per-group flags, tickets and counters
 *    in the workspace and update the state in place.
 *  - Asynchronous on the caller's stream (`stream` is a cudaStream_t; NULL =
 *    legacy default stream). Nothing synchronises except nosa_check_device.
 *  - The caller owns all memory: device buffers (any allocator) and, for
 *    offload, pinned host buffers (cudaHostAlloc / torch pin_memory), which are
 *    device-accessible under unified addressing. The library allocates nothing.
 *  - Every pointer must be 16-byte aligned. bf16 tensors are passed as raw
 *    16-bit patterns (uint16_t).
 *  - Device-side faults (a corrupt block table, a selected block that is not
 *    resident, a bounded wait that ran out) do not trap: the kernel records a
 *    bit in state->err, skips the bad access and returns. nosa_check_device
 *    reads that word.
 *  - A group is gi = b * Hkv + g; query head h of batch b belongs to group
 *    b * Hkv + h / G with G = Hq / Hkv.
 *
 * Notation: bs = block_size, s = sub_block, N = ceil(L / bs) blocks and
 * M = ceil(L / s) sub-blocks for a context of L tokens, k = k_q + k_e,
 * W = ceil(max_blocks / 32), max_sub = max_blocks * bs / s.
 */
#ifndef NOSA_H
#define NOSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nosa_status {
  NOSA_OK = 0,
  NOSA_EINVAL = 1,   /* bad shape, size, alignment or pointer kind; nothing launched */
  NOSA_ENOMEM = 2,   /* caller's workspace smaller than nosa_workspace_size */
  NOSA_ECUDA = 3,    /* a CUDA runtime call failed (launch, attribute query) */
  NOSA_EDEVICE = 4,  /* nosa_check_device: a kernel recorded a fault in state->err */
  NOSA_ETIMEOUT = 5  /* nosa_check_device: a bounded device wait ran out */
} nosa_status;

/* Device error word bits (state->err). */
#define NOSA_ERR_BLOCK_TABLE 0x1u  /* page index out of range or selected block not resident */
#define NOSA_ERR_SEL 0x2u          /* selected index outside [0, N) */
#define NOSA_ERR_NO_VICTIM 0x4u    /* residency: fewer evictable blocks than misses */
#define NOSA_ERR_TIMEOUT 0x8u      /* an mbarrier wait exceeded its time limit */
#define NOSA_ERR_FULL 0x10u        /* append beyond max_blocks * block_size tokens */
#define NOSA_ERR_INIT 0x20u        /* state init: more resident blocks than slots */

typedef struct nosa_config {
  int32_t B, Hq, Hkv;     /* batch, query heads, KV heads; G = Hq / Hkv in {1, 2, 4, 8} */
  int32_t d;              /* head dim: 64 or 128 */
  int32_t block_size;     /* tokens per block (selection unit, one page): 32, 64 or 128 */
  int32_t sub_block;      /* tokens per pooling sub-block: 8, 16 or 32, dividing block_size */
  int32_t k_q, k_e;       /* query-aware and query-agnostic budgets, k = k_q + k_e >= 1 */
  int32_t max_blocks;     /* blocks per group the cache can hold (<= 8192, >= k) */
  int32_t slots;          /* HBM pages per group: == max_blocks without host pools,
                             else in [k + 2, max_blocks] */
  int32_t n_score_rows;   /* G: score with the group's query heads; 1: one forecast row */
  int32_t attn_split;     /* selected blocks per attention CTA; 0 = automatic */
  float scale;            /* sigma, the softmax scale (1/sqrt(d) for standard attention) */
  int32_t score_mode;     /* scoring variant bits, 0 = the NOSA pool (sub-block means, mean of
                             the rows' raw logits). NOSA_SCORE_WINDOW: units are windows of two
                             sub-blocks at a stride of one (SparDA's (32, 16) inference window
                             at sub_block 16, gist.science/de/paper/2606.04511, section 2
                             "Trainingsstrategie"); NOSA_SCORE_SOFTMAX: per scoring row a softmax
                             over all units, summed over the rows (needs n_score_rows <= 8).
                             A block's score is the max over the units starting in it. Variants
                             run only in nosa_step and nosa_plan_ahead. */
  float stop_tau;         /* > 0: S2O's monotone-gain early stop (gist.science/it/paper/2602.22575,
                             "Regola di Arresto Anticipato") in nosa_step: each query head visits
                             the selected blocks in decreasing block score (ties: lower index) and
                             stops after the first block whose gain in softmax mass is below
                             stop_tau times the mass accumulated so far, that block included.
                             0: attend every selected block. Needs k <= 1024. */
  int32_t kc_bf16;        /* 1: state->kc holds bf16 sub-block means (each mean is summed in fp32 in
                             token order, divided in fp32 and rounded to nearest even), half the
                             score kernel's bytes; 0: fp32 means. */
  int32_t wait_us;        /* limit of every bounded device wait (a per-group flag, an mbarrier), in
                             microseconds from the waiting kernel's start, in [0, 60000000];
                             0 = 4 s. A wait that runs out sets NOSA_ERR_TIMEOUT and the kernel
                             returns; nosa_check_device then reports NOSA_ETIMEOUT. */
} nosa_config;

#define NOSA_SCORE_WINDOW 1
#define NOSA_SCORE_SOFTMAX 2

/*
 * Decode state: caller-allocated buffers, sized by nosa_state_sizes.
 * Pools are paged: page p holds one block of one group, [block_size][d] bf16
 * row-major. Without host pools page gi * max_blocks + j holds block j of group
 * gi (the caller writes the prefill there before nosa_state_init). With host
 * pools the host copy is the full backing store, [B*Hkv][max_blocks][bs][d],
 * and the block table maps resident blocks to HBM pages gi * slots + z.
 */
typedef struct nosa_state {
  int32_t* seq_len;       /* [B*Hkv] tokens in the cache */
  float* kc;              /* [B*Hkv][max_sub][d] sub-block mean keys: fp32, or bf16 with kc_bf16 */
  uint32_t* prev_sel;     /* [B*Hkv][W] bitmask of S(t-1) */
  uint32_t* alive;        /* [B*Hkv][W] bitmask of A(t-1), blocks still eligible for Gamma_e */
  int32_t* last_used;     /* [B*Hkv][max_blocks] context length when last needed (LRU stamp) */
  int32_t* block_table;   /* [B*Hkv][max_blocks] HBM page, or -1 when only on the host */
  int32_t* slot_owner;    /* [B*Hkv][slots] block held by HBM slot z, or -1 */
  uint16_t* k_pool;       /* [B*Hkv*slots][bs][d] bf16, device */
  uint16_t* v_pool;
  uint16_t* host_k;       /* [B*Hkv][max_blocks][bs][d] bf16, pinned host; NULL = all in HBM */
  uint16_t* host_v;
  uint32_t* err;          /* [1] device error word (NOSA_ERR_* bits) */
} nosa_state;

typedef struct nosa_sizes {  /* bytes of each nosa_state buffer */
  size_t seq_len, kc, prev_sel, alive, last_used, block_table, slot_owner, k_pool, v_pool,
      host_k, host_v, err;
} nosa_sizes;

/* Validates cfg; fills the byte size of every state buffer. */
nosa_status nosa_state_sizes(const nosa_config* cfg, nosa_sizes* out);

/* Scratch bytes the step needs (block scores, counters, copy lists, split-K partials). */
nosa_status nosa_workspace_size(const nosa_config* cfg, size_t* bytes);

/* Zeroes the workspace (its counters must start at zero). Call once after allocating it,
 * and again after nosa_check_device reported a fault. */
nosa_status nosa_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/*
 * Builds the decode state from the prefill. prefill_len: device int32 [B], tokens
 * already written (per batch entry; may differ, may be 0). Without host pools the
 * prefill is read from the device pools; with host pools from the host copy, and
 * `resident` (device uint8 [B*Hkv][max_blocks], nonzero = start in HBM, at most
 * `slots` per group) picks the blocks copied to HBM slots 0, 1, ... in ascending
 * block order. Sets kc = sub-block means, S(-1) = A(-1) = all prefill blocks
 * (NOSA, "Seleccion Independiente de la Consulta"), last_used = 0, err = 0.
 */
nosa_status nosa_state_init(const nosa_config* cfg, const nosa_state* st, const int32_t* prefill_len,
                            const uint8_t* resident, void* workspace, size_t ws_bytes, void* stream);

/*
 * Append one token per group: k_new, v_new device bf16 [B*Hkv][d] become token
 * L-1 (L = seq_len + 1), written to the tail page when it is resident and always
 * through to the host copy when there is one; kc of the tail sub-block is
 * recomputed as the fp32 mean of its present tokens; seq_len += 1.
 * (NOSA, "Layout de Memoria Optimizado": KV kept in minimal block units.)
 */
nosa_status nosa_append(const nosa_config* cfg, const nosa_state* st, const uint16_t* k_new,
                        const uint16_t* v_new, void* stream);

/*
 * Two-stage pooled block scores (NOSA, "Implementacion Basada en Bloques"):
 *   u_i = sigma * mean_r (rows_r . kc_i),  s_j = max over the present sub-blocks i of block j.
 * score_rows: device bf16 [B*Hkv][n_score_rows][d] (for n_score_rows = G this is q
 * [B][Hq][d] itself). block_scores: device fp32 [B*Hkv][max_blocks]; entries >= N
 * are written -inf. No softmax: selection runs on pre-exponential scores.
 */
nosa_status nosa_score_blocks(const nosa_config* cfg, const nosa_state* st, const uint16_t* score_rows,
                              float* block_scores, void* stream);

/*
 * Dual selection (NOSA, "Seleccion Sensible a la Consulta", "Seleccion Independiente
 * de la Consulta", "Garantia de Localidad"):
 *   C_e = S(t-1) & A(t-1); Gamma_e = top-min(k_e, |C_e|) of evict_scores over C_e;
 *   A(t) = A(t-1) minus (C_e minus Gamma_e);
 *   Gamma_q = top-min(k - |Gamma_e|, N - |Gamma_e|) of block_scores over [0, N) minus Gamma_e;
 *   S(t) = Gamma_e + Gamma_q.
 * Higher score first, equal scores (after -0 -> +0) to the lower index.
 * evict_scores: device fp32 [B*Hkv][max_blocks]. sel: device int32 [B*Hkv][k], S(t)
 * ascending, padded with -1. Updates prev_sel and alive.
 */
nosa_status nosa_select(const nosa_config* cfg, const nosa_state* st, const float* block_scores,
                        const float* evict_scores, int32_t* sel, void* stream);

/*
 * Residency and gather (NOSA, "Layout de Memoria Optimizado" set differences and
 * "Comunicacion de Alto Ancho de Banda" UVA transfer kernels): misses = (S(t) +
 * tail block) minus resident blocks; slots = free slots ascending, then the least
 * recently used resident blocks outside S(t) + tail (ties to the lower index) in
 * ascending block order; each miss (ascending) gets the next slot, its K and V
 * pages are copied from the host copy with 16-byte loads over UVA, the block table
 * and slot owners are updated, last_used = L for S(t) + tail. miss_count: device
 * int32 [B*Hkv] (pages fetched). Without host pools it writes zeros.
 */
nosa_status nosa_gather(const nosa_config* cfg, const nosa_state* st, const int32_t* sel,
                        int32_t* miss_count, void* workspace, size_t ws_bytes, void* stream);

/*
 * Split-K flash-decoding over the selected blocks (spec step; online-softmax
 * state (m, l, acc) and its merge as in S2O's two-pass kernel, gist.science/it/paper/
 * 2602.22575, "Implementazione del Kernel"):
 *   out[b][h] = sum over tokens tau < L of blocks in sel of softmax(sigma q_h . K_tau) V_tau.
 * q: device bf16 [B][Hq][d]; sel as from nosa_select (every block resident);
 * out: device fp32 [B][Hq][d].
 */
nosa_status nosa_decode_attn(const nosa_config* cfg, const nosa_state* st, const uint16_t* q,
                             const int32_t* sel, float* out, void* workspace, size_t ws_bytes,
                             void* stream);

/*
 * One whole decode step: append -> score -> select -> gather -> attention, in two kernels
 * (three with host pools; nosa_step_launches reports the count). score_rows NULL = score
 * with q (requires n_score_rows == G). events: NULL, or 4 cudaEvent_t recorded on the stream
 * before the first kernel and after each of score/select, gather and attention (profiling).
 */
nosa_status nosa_step(const nosa_config* cfg, const nosa_state* st, const uint16_t* q,
                      const uint16_t* score_rows, const uint16_t* k_new, const uint16_t* v_new,
                      const float* evict_scores, int32_t* sel, float* out, int32_t* miss_count,
                      void* workspace, size_t ws_bytes, void* stream, void* const* events);

/*
 * How many kernels one nosa_step launches for this configuration and state: 2 (score +
 * selection, attention) or 3 with host pools (score + selection, page copies, attention).
 * Launches nothing; the state is checked as nosa_step checks it (host pools: one
 * cudaPointerGetAttributes each). kernels: host int32, written on success. Errors:
 * NOSA_EINVAL for a bad configuration or state, or a NULL kernels.
 */
nosa_status nosa_step_launches(const nosa_config* cfg, const nosa_state* st, int32_t* kernels);

/*
 * Launch geometry of the step's kernels for this configuration on a GPU with `sms` SMs on which
 * `attn_ctas_per_sm` attention CTAs are resident at once (two on a B200 with 64-token blocks and
 * d = 128), as nosa_step (given no events) chooses it:
 *   score_chunk        sub-blocks per score CTA: the fewest equal chunks of at most 384 that
 *                      cover the group's sub-blocks, rounded up to 64, and for small batches at
 *                      least about three score CTAs per SM in all (chunks down to 64);
 *   score_ctas         score CTAs (groups x chunks per group);
 *   attn_tasks_per_cta (group, block) tasks per attention CTA: attn_split when set; with host
 *                      pools the smallest width the 16 partial slots per group allow; otherwise a
 *                      divisor of k near one CTA per resident slot, or one CTA per group when a
 *                      group's selected K and V pages total at most 512 KB and the groups number
 *                      between a quarter of the SMs and one wave; with early stop one CTA per
 *                      group;
 *   attn_ctas          attention CTAs.
 * host_pools: nonzero for a state with host pools. No CUDA call. Errors: NOSA_EINVAL for a bad
 * configuration, sms or attn_ctas_per_sm < 1, or a NULL out.
 */
typedef struct nosa_geometry {
  int32_t score_chunk;
  int32_t score_ctas;
  int32_t attn_tasks_per_cta;
  int32_t attn_ctas;
} nosa_geometry;

nosa_status nosa_step_geometry(const nosa_config* cfg, int32_t host_pools, int32_t sms,
                               int32_t attn_ctas_per_sm, nosa_geometry* out);

/*
 * Lookahead decoding (SparDA, gist.science/de/paper/2606.04511, section 2: "Trainierbare
 * Lookahead Sparse-Selektion", "Asynchrones Prefetching mit persistentem UVA-Kernel"): the
 * blocks a step attends are chosen from a forecast row before the step's query exists, so
 * their host -> HBM copies can run while other work (e.g. the previous layer) computes.
 * Three calls per step and state, in this order:
 *
 * nosa_plan_ahead scores the cache as it stands (no append) with score_rows
 * ([B*Hkv][n_score_rows][d] bf16, e.g. one forecast row per group), runs the dual selection
 * (sel [B*Hkv][k] and miss_count [B*Hkv] as in nosa_step) and, with host pools, the
 * residency plan.
 *
 * nosa_prefetch (host pools; a no-op without) copies the planned pages host -> HBM over UVA,
 * group after group. It may run on another stream once nosa_plan_ahead has completed.
 *
 * nosa_attend appends k_new / v_new ([B*Hkv][d] bf16) and attends q ([B][Hq][d] bf16) over
 * the blocks sel chose (out [B][Hq][d] fp32). On the GPU each group first acquires its
 * "pages in place" flag (bounded wait, NOSA_ERR_TIMEOUT on expiry). It must be issued after
 * nosa_plan_ahead has completed; issue it after nosa_prefetch has completed too (same
 * stream, or an event), so that its CTAs never sit on the SMs waiting for copies.
 *
 * Rules: the three calls of a step use the same state, workspace and sel, and no other call
 * on that state and workspace comes between them. The triple computes what the oracle's
 * lookahead order defines: select and plan at length L, append (L + 1), attend; a block the
 * append creates is not a candidate of the step. Needs a non-empty cache (L >= 1).
 */
nosa_status nosa_plan_ahead(const nosa_config* cfg, const nosa_state* st, const uint16_t* score_rows,
                            const float* evict, int32_t* sel, int32_t* miss_count, void* workspace,
                            size_t ws_bytes, void* stream);
nosa_status nosa_prefetch(const nosa_config* cfg, const nosa_state* st, void* workspace, size_t ws_bytes,
                          void* stream);
nosa_status nosa_attend(const nosa_config* cfg, const nosa_state* st, const uint16_t* q,
                        const uint16_t* k_new, const uint16_t* v_new, const int32_t* sel, float* out,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * No-allocation variant of nosa_decode_attn (the pages have no counterpart: this is an
 * integration aid). Some callers cannot call cudaMalloc when they run attention: plugins
 * inside a host framework that owns all device memory, or a latency-bound serving loop that
 * must not allocate or synchronise. This entry point
 * computes exactly what nosa_decode_attn computes but takes no workspace: its scratch (the
 * split-K partials and the per-group counters) lives in a static device array of 8 MiB
 * inside the library, which every GPU that loads the library keeps until the process exits.
 * Limit: B*Hkv * (16 * G * (d + 2) * 4 bytes, rounded up to 256) plus B*Hkv * 4 bytes must
 * fit in 8 MiB (about 250 groups at G = 4, d = 128); larger configurations get NOSA_ENOMEM and
 * must use nosa_decode_attn with a workspace. Allocates nothing: no cudaMalloc, no cudaFree.
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture. Every call
 * shares the one array: it zeroes the counters it needs on `stream` before the kernel, and
 * calls whose kernels overlap on the GPU (other streams, other threads) race on the scratch.
 */
nosa_status nosa_decode_attn_noalloc(const nosa_config* cfg, const nosa_state* st, const uint16_t* q,
                                     const int32_t* sel, float* out, void* stream);

/*
 * Measurement helper, not a step of the decode path (the pages give no such call): copies
 * `bytes` of pinned, device-mapped host memory at `host` to device memory at `dev` with
 * 16-byte loads over UVA, the access the gather kernel makes, on `ctas` CTAs of 256 threads
 * (0: four per SM). The time of this call is the PCIe read ceiling the gather is measured
 * against. host and dev must be 16-byte aligned and bytes a multiple of 16; NOSA_EINVAL
 * otherwise, or when host is not pinned, device-mapped host memory. Asynchronous on stream.
 */
nosa_status nosa_uva_read_probe(const void* host, void* dev, size_t bytes, int ctas, void* stream);

/*
 * Early stop bookkeeping: copies, for the last nosa_step run with stop_tau > 0 on this
 * workspace, the number of blocks each query head visited into used (device, [B][Hq] int32,
 * 16-byte aligned). Asynchronous on stream.
 */
nosa_status nosa_stop_counts(const nosa_config* cfg, const void* workspace, size_t ws_bytes,
                             int32_t* used, void* stream);

/* Synchronises the stream, reads state->err into *err_out (may be NULL):
 * NOSA_OK, NOSA_EDEVICE or NOSA_ETIMEOUT. */
nosa_status nosa_check_device(const nosa_state* st, void* stream, uint32_t* err_out);

const char* nosa_status_string(nosa_status s);
const char* nosa_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* NOSA_H */
