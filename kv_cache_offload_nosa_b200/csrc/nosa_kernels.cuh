// Score / append / select / gather / init kernels of the NOSA decode step.
//
// NOSA: Native and Offloadable Sparse Attention (technical summary at
// gist.science/es/paper/2510.13602): "Metodologia" 1, "Implementacion Basada en Bloques"
// (each sub-block is represented by its mean key; a block's score is the max over its
// sub-blocks' scores) and 2, "Layout de Memoria
// Optimizado" (KV kept in minimal block units; set differences decide the pages to swap)
// and "Comunicacion de Alto Ancho de Banda" (UVA copy kernels for the host -> HBM pages).
//
// score_kernel streams the fp32 sub-block mean keys (kc) of every group once:
// HBM-bound at one FMA per 4 bytes, so it is written for coalesced 16-byte
// loads (each warp covers whole sub-blocks with 128-byte segments), a grid of
// B*Hkv x ceil(max_sub/256) CTAs of 256 threads, and warp-shuffle reductions.
// Fused form: the CTA owning the tail sub-block appends the new token first,
// and the last CTA of each group to finish (atomic ticket, no spinning) runs
// the dual selection and, with host pools, the residency plan.
#pragma once

#include <type_traits>

#include "nosa_select.cuh"

namespace nosa {

constexpr int kScoreThreads = 256;
constexpr int kChunkAlign = 64;  // a score CTA's sub-block count is a multiple of this

struct StepArgs {
  // scoring
  const uint16_t* rows;   // [B*Hkv][R][d] bf16
  int R;
  float* kc;
  float* block_scores;    // [B*Hkv][max_blocks]
  int32_t* seq_len;
  int max_blocks, max_sub, bs, s, slots;
  float scale;
  long long total_pages;
  // append
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* k_pool;
  uint16_t* v_pool;
  uint16_t* host_k;
  uint16_t* host_v;
  int32_t* block_table;
  // selection
  const float* evict;
  uint32_t* prev_sel;
  uint32_t* alive;
  int32_t* sel;
  int k_q, k_e;
  // residency
  int32_t* slot_owner;
  int32_t* last_used;
  int2* copy_list;
  int copy_stride;
  int32_t* copy_count;
  int32_t* miss_count;
  uint32_t* counters;
  uint32_t* ge_mask;      // [B*Hkv][W] Gamma_e handed from chunk 0 to the last chunk
  uint32_t* sel_flag;     // [B*Hkv * kFlagStride] set (release) once a group's selection is published, or NULL
  uint32_t* err;
  int append;             // fused score kernel: 1 appends the step's token first, 0 scores the
                          // cache as it stands (lookahead planning)
  const uint32_t* ready;  // append_kernel: per-group flags to acquire before writing, or NULL
  int kc16;               // kc holds bf16 means (else fp32)
  int mode;               // scoring variant bits (1 windows, 2 per-row softmax); 0 = NOSA pool
  float* units;           // variants: per-sub-block values [B*Hkv][rows][max_sub] (workspace)
  int chunk;              // sub-blocks per score CTA (a multiple of kChunkAlign)
  unsigned long long wait_ns;  // limit of the bounded waits (append_kernel's flag)
  // early publication of the query-agnostic set (fused step with per-group flags), or NULL:
  int32_t* att_list;      // [B*Hkv][k] attention order: Gamma_e ascending, Gamma_q ascending, -1
  uint32_t* e_flag;       // [B*Hkv * kFlagStride]: [0] set once Gamma_e is in att_list and the
                          // step's token is in place, [1] the context length L after the
                          // append, [2] the early part's length, [3] parties done (0..2)
};

constexpr int kMaxSoftRows = 8;  // scoring rows the per-row softmax variant supports

// Block scores of the scoring variants, computed by the last CTA of a group from the
// per-sub-block values its chunks left in a.units (softmax: sigma q_r . kbar_i per row r;
// otherwise the mean over the rows). The unit starting at sub-block i is that sub-block or,
// with windows, the window of sub-blocks i and i+1: its value is the present-token-weighted
// mean of theirs (the logit of the window's mean key, by linearity). Softmax: per row over
// all units, then the sum over the rows. Block score = max over the units starting in it.
// (SparDA, gist.science/de/paper/2606.04511, section 2: the (32, 16) inference window and the
// per-head softmax scoring its compact indexer removes.)
template <bool SOFT>
__device__ void variant_block_scores(const StepArgs& a, int gi, int L, int M, int N, float* red) {
  const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nw = nth >> 5;
  const bool win = (a.mode & 1) != 0;
  constexpr bool soft = SOFT;
  const int Ru = soft ? a.R : 1;
  const int spb = a.bs / a.s;
  const float* v = a.units + (size_t)gi * Ru * a.max_sub;
  auto unit = [&](int r, int i) -> float {
    const float* vr = v + (size_t)r * a.max_sub;
    const float x0 = __ldcg(vr + i);
    if (!win || i + 1 >= M) return x0;
    const int n0 = min(a.s, L - i * a.s), n1 = min(a.s, L - (i + 1) * a.s);
    return (n0 * x0 + n1 * __ldcg(vr + i + 1)) / (float)(n0 + n1);
  };
  float* mx = red;                    // [kMaxSoftRows]
  float* den = red + kMaxSoftRows;    // [kMaxSoftRows]
  float* part = red + 2 * kMaxSoftRows;  // [kMaxSoftRows][nw]
  if constexpr (SOFT) {
    for (int pass = 0; pass < 2; ++pass) {
      float acc[kMaxSoftRows];
#pragma unroll
      for (int r = 0; r < kMaxSoftRows; ++r) acc[r] = pass == 0 ? -INFINITY : 0.f;
#pragma unroll 4
      for (int i = tid; i < M; i += nth) {
#pragma unroll
        for (int r = 0; r < kMaxSoftRows; ++r)
          if (r < Ru) {
            const float x = unit(r, i);
            acc[r] = pass == 0 ? fmaxf(acc[r], x) : acc[r] + expf(x - mx[r]);
          }
      }
#pragma unroll
      for (int r = 0; r < kMaxSoftRows; ++r) {
        if (r >= Ru) break;
        float x = acc[r];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          const float y = __shfl_xor_sync(0xffffffffu, x, o);
          x = pass == 0 ? fmaxf(x, y) : x + y;
        }
        if (lane == 0) part[r * nw + warp] = x;
      }
      __syncthreads();
      if (tid < Ru) {
        float x = pass == 0 ? -INFINITY : 0.f;
        for (int w = 0; w < nw; ++w) x = pass == 0 ? fmaxf(x, part[tid * nw + w]) : x + part[tid * nw + w];
        (pass == 0 ? mx : den)[tid] = x;
      }
      __syncthreads();
    }
  }
  for (int j = tid; j < a.max_blocks; j += nth) {
    float m = -INFINITY;
    if (j < N) {
      const int e = min((j + 1) * spb, M);
      for (int i = j * spb; i < e; ++i) {
        float p;
        if constexpr (SOFT) {
          p = 0.f;
          for (int r = 0; r < Ru; ++r) p += expf(unit(r, i) - mx[r]) / den[r];
        } else {
          p = unit(0, i);
        }
        m = fmaxf(m, p);
      }
    }
    a.block_scores[(size_t)gi * a.max_blocks + j] = m;
  }
  __threadfence();
  __syncthreads();
}

// Append token pos = len0 of group gi (all threads of the CTA take part).
template <int D>
__device__ void append_token(const StepArgs& a, int gi, int len0) {
  const int pos = len0;
  const int jb = pos / a.bs, r = pos % a.bs, sb = pos / a.s;
  int page = a.block_table[(size_t)gi * a.max_blocks + jb];
  if (page >= a.total_pages || (page < 0 && !a.host_k)) {
    if (threadIdx.x == 0) set_err(a.err, NOSA_ERR_BLOCK_TABLE);
    page = -1;
  }
  const size_t hbase = ((size_t)gi * a.max_blocks + jb) * a.bs;
  const int t0 = sb * a.s;
  for (int x = threadIdx.x; x < D; x += blockDim.x) {
    const uint16_t kx = a.k_new[(size_t)gi * D + x];
    const uint16_t vx = a.v_new[(size_t)gi * D + x];
    float sum = 0.f;
    if (page >= 0 || a.host_k) {
#pragma unroll 8
      for (int tau = t0; tau < pos; ++tau) {
        const int rr = tau - jb * a.bs;
        const uint16_t* src = (page >= 0) ? a.k_pool + ((size_t)page * a.bs + rr) * D
                                          : a.host_k + (hbase + rr) * D;
        sum += bf16_bits_to_f32(src[x]);
      }
    }
    sum += bf16_bits_to_f32(kx);
    if (page >= 0) {
      a.k_pool[((size_t)page * a.bs + r) * D + x] = kx;
      a.v_pool[((size_t)page * a.bs + r) * D + x] = vx;
    }
    if (a.host_k) {
      a.host_k[(hbase + r) * D + x] = kx;
      a.host_v[(hbase + r) * D + x] = vx;
    }
    const float mean = __fdiv_rn(sum, (float)(pos - t0 + 1));
    const size_t ki = ((size_t)gi * a.max_sub + sb) * D + x;
    if (a.kc16) reinterpret_cast<__nv_bfloat16*>(a.kc)[ki] = __float2bfloat16_rn(mean);
    else a.kc[ki] = mean;
  }
}

// VARIANT: the scoring variants (a.mode != 0; 1: mean of the rows, windows; 2: per-row
// softmax); the chunks leave per-sub-block values in a.units and the group's last CTA turns
// them into block scores (fused launches only).
// KC16: kc holds bf16 means (one 16-byte load carries 8 of them; the lanes of a sub-block row
// still read it in contiguous 128-byte pieces).
template <int D, bool FUSED, int VARIANT = 0, bool KC16 = false>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(StepArgs a) {
  constexpr int LPS = D / 16;        // lanes per sub-block (16 values each)
  constexpr int SPW = 32 / LPS;      // sub-blocks per warp pass
  constexpr int PASS = SPW * (kScoreThreads / 32);
  __shared__ float qbar[D];
  __shared__ int s_last;
  __shared__ float vred[VARIANT ? 2 * kMaxSoftRows + kMaxSoftRows * (kScoreThreads / 32) : 1];
  extern __shared__ __align__(16) uint8_t dsm[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gi = blockIdx.y, c = blockIdx.x;
  const int i0 = c * a.chunk;
  // dynamic shared memory: [selection scratch (fused)] [this chunk's sub-block values]
  float* su = reinterpret_cast<float*>(dsm + (FUSED ? score_su_offset(a.max_blocks) : 0));
  const int sub = lane / LPS, part = lane % LPS;
  using Vec = typename std::conditional<KC16, uint4, float4>::type;
  constexpr int NV = KC16 ? 2 : 4;          // 16-byte loads per lane and sub-block row
  constexpr int EV = KC16 ? 8 : 4;          // values per 16-byte load
  constexpr int VPR = D / EV;               // 16-byte vectors per row
  const Vec* kcg = reinterpret_cast<const Vec*>(
      reinterpret_cast<const uint8_t*>(a.kc) + (size_t)gi * a.max_sub * D * (KC16 ? 2 : 4));

  if (FUSED) griddep_launch_dependents();  // the next kernel may start its prologue
  // first batch of kc loads goes out before anything that depends on seq_len
  const int icap = min(i0 + a.chunk, a.max_sub);
  int base = i0 + warp * SPW;
  Vec va[NV], vb[NV];
  auto load_batch = [&](int bse, int lim, Vec* xa, Vec* xb) {
    const int ia = bse + sub, ib = bse + PASS + sub;
    Vec z;
    memset(&z, 0, sizeof(z));
#pragma unroll
    for (int jj = 0; jj < NV; ++jj) {
      const int p4 = part + LPS * jj;
      xa[jj] = (ia < lim) ? __ldcs(kcg + (size_t)ia * VPR + p4) : z;
      xb[jj] = (ib < lim) ? __ldcs(kcg + (size_t)ib * VPR + p4) : z;
    }
  };
  load_batch(base, icap, va, vb);

  const int len0 = a.seq_len[gi];
  int L = len0;
  if (FUSED && a.append) {
    if (len0 < a.max_blocks * a.bs) L = len0 + 1;
    else if (c == 0 && tid == 0) set_err(a.err, NOSA_ERR_FULL);
  }
  const int M = (L + a.s - 1) / a.s;
  const int N = (L + a.bs - 1) / a.bs;
  const int spb = a.bs / a.s;
  const int i1 = min(i0 + a.chunk, M);
  const int Wmax = (a.max_blocks + 31) / 32;

  // The query-agnostic selection needs no block score: chunk 0 runs it while the other chunks
  // stream. With early publication its blocks can be attended before the query-aware half is
  // known (NOSA, "Seleccion Independiente de la Consulta": Gamma_e depends on the eviction
  // scores only), once the step's token is in place too: chunk 0 and the chunk that appends
  // each count themselves done, and the second publishes. Only Gamma_e's blocks already in
  // HBM go early: Gamma_e lies in S(t-1), which the previous step made resident, but the
  // first step after set-up starts from S(-1) = every prefill block and only the initial
  // residency.
  const int c_app = (FUSED && L > len0) ? (len0 / a.s) / a.chunk : -1;
  const bool parties2 = c_app > 0;  // chunk 0 and another chunk share the publication
  if (FUSED && c == c_app) {
    append_token<D>(a, gi, len0);
    __syncthreads();
    load_batch(base, icap, va, vb);  // the tail sub-block's mean just changed
  }
  if (FUSED && c == 0) {
    const SelSmem S = sel_smem_carve(dsm, a.max_blocks);
    select_evict(S, a.evict + (size_t)gi * a.max_blocks, a.prev_sel + (size_t)gi * Wmax,
                 a.alive + (size_t)gi * Wmax, a.ge_mask + (size_t)gi * Wmax, N, a.k_e, Wmax);
    if (a.e_flag) {
      const int W = (N + 31) / 32;
      resident_bits(S.ge, S.m2, a.host_k ? a.block_table + (size_t)gi * a.max_blocks : nullptr, W);
      const int ne = sel_compact(S, S.m2, W, a.att_list + (size_t)gi * (a.k_q + a.k_e));
      if (tid == 0) a.e_flag[(size_t)gi * kFlagStride + 2] = static_cast<uint32_t>(ne);
    }
  }
  if (FUSED && a.e_flag && (c == 0 || c == c_app)) {
    __syncthreads();  // this CTA's part (Gamma_e's list, or the appended token) is written
    if (tid == 0) {
      uint32_t* ef = a.e_flag + (size_t)gi * kFlagStride;
      __threadfence();
      const bool second = !parties2 || atomicAdd(ef + 3, 1u) == 1u;
      if (second) {
        __threadfence();
        ef[1] = static_cast<uint32_t>(L);
        st_release_gpu(ef, 1u);
      }
    }
  }
  for (int x = tid; x < D; x += kScoreThreads) {
    const uint16_t* r = a.rows + (size_t)gi * a.R * D + x;
    float sacc = 0.f;
    for (int rr = 0; rr < a.R; ++rr) sacc += bf16_bits_to_f32(r[(size_t)rr * D]);
    qbar[x] = a.scale * sacc / (float)a.R;
  }
  __syncthreads();
  constexpr bool soft = VARIANT == 2;

  if (soft && i0 < i1) {
    // per-row logits sigma q_r . kbar_i: one sub-block row per LPR lanes (one float4 each),
    // the group's rows in registers; warp-uniform trip count so the shuffles see full warps
    constexpr int LPR = D / 4, RPW = 32 / LPR, WROWS = RPW * (kScoreThreads / 32);
    const int sub2 = lane / LPR, p2 = lane % LPR;
    float4 qv[kMaxSoftRows];
#pragma unroll
    for (int r = 0; r < kMaxSoftRows; ++r) {
      qv[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < a.R) {
        const uint16_t* qr = a.rows + ((size_t)gi * a.R + r) * D + 4 * p2;
        qv[r] = make_float4(a.scale * bf16_bits_to_f32(qr[0]), a.scale * bf16_bits_to_f32(qr[1]),
                            a.scale * bf16_bits_to_f32(qr[2]), a.scale * bf16_bits_to_f32(qr[3]));
      }
    }
    constexpr int RF = 4;  // rows in flight per warp
    for (int b0 = i0 + warp * RPW; b0 < i1; b0 += RF * WROWS) {
      float4 x[RF];
#pragma unroll
      for (int f = 0; f < RF; ++f) {
        const int i = b0 + f * WROWS + sub2;
        x[f] = make_float4(0, 0, 0, 0);
        if (i < i1) {
          if constexpr (KC16) {
            const uint2 w = __ldcs(reinterpret_cast<const uint2*>(kcg) + (size_t)i * (D / 4) + p2);
            x[f] = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                               __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
          } else {
            x[f] = __ldcs(reinterpret_cast<const float4*>(kcg) + (size_t)i * (D / 4) + p2);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kMaxSoftRows; ++r) {
        if (r >= a.R) break;
        float z[RF];
#pragma unroll
        for (int f = 0; f < RF; ++f)
          z[f] = qv[r].x * x[f].x + qv[r].y * x[f].y + qv[r].z * x[f].z + qv[r].w * x[f].w;
#pragma unroll
        for (int o = LPR / 2; o >= 1; o >>= 1)
#pragma unroll
          for (int f = 0; f < RF; ++f) z[f] += __shfl_xor_sync(0xffffffffu, z[f], o);
        float* ur = a.units + ((size_t)gi * a.R + r) * a.max_sub;
#pragma unroll
        for (int f = 0; f < RF; ++f) {
          const int i = b0 + f * WROWS + sub2;
          if (p2 == 0 && i < i1) ur[i] = z[f];
        }
      }
    }
  }
  if (!soft && i0 < i1) {
    float qr[16];  // this lane's 16 values of qbar, in the order of its loads
#pragma unroll
    for (int jj = 0; jj < NV; ++jj) {
      const int p4 = part + LPS * jj;
#pragma unroll
      for (int e = 0; e < EV; ++e) qr[EV * jj + e] = qbar[EV * p4 + e];
    }
    for (; base < i1; base += 2 * PASS) {
      Vec na[NV], nb[NV];
      load_batch(base + 2 * PASS, i1, na, nb);  // next batch in flight during this one
      const int ia = base + sub, ib = base + PASS + sub;
      float da = 0.f, db = 0.f;
#pragma unroll
      for (int jj = 0; jj < NV; ++jj) {
        if constexpr (KC16) {
          const uint32_t wa[4] = {va[jj].x, va[jj].y, va[jj].z, va[jj].w};
          const uint32_t wb[4] = {vb[jj].x, vb[jj].y, vb[jj].z, vb[jj].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            da = fmaf(qr[8 * jj + 2 * h], __uint_as_float(wa[h] << 16), da);
            da = fmaf(qr[8 * jj + 2 * h + 1], __uint_as_float(wa[h] & 0xffff0000u), da);
            db = fmaf(qr[8 * jj + 2 * h], __uint_as_float(wb[h] << 16), db);
            db = fmaf(qr[8 * jj + 2 * h + 1], __uint_as_float(wb[h] & 0xffff0000u), db);
          }
        } else {
          da = fmaf(qr[4 * jj + 0], va[jj].x, da);
          da = fmaf(qr[4 * jj + 1], va[jj].y, da);
          da = fmaf(qr[4 * jj + 2], va[jj].z, da);
          da = fmaf(qr[4 * jj + 3], va[jj].w, da);
          db = fmaf(qr[4 * jj + 0], vb[jj].x, db);
          db = fmaf(qr[4 * jj + 1], vb[jj].y, db);
          db = fmaf(qr[4 * jj + 2], vb[jj].z, db);
          db = fmaf(qr[4 * jj + 3], vb[jj].w, db);
        }
      }
#pragma unroll
      for (int o = LPS / 2; o >= 1; o >>= 1) {
        da += __shfl_xor_sync(0xffffffffu, da, o);
        db += __shfl_xor_sync(0xffffffffu, db, o);
      }
      if (part == 0) {
        if (ia < i1) su[ia - i0] = da;
        if (ib < i1) su[ib - i0] = db;
      }
#pragma unroll
      for (int jj = 0; jj < NV; ++jj) {
        va[jj] = na[jj];
        vb[jj] = nb[jj];
      }
    }
  }
  __syncthreads();
  if (VARIANT && !soft) {
    // the mean-of-rows values of the chunk's sub-blocks, for the group's last CTA
    for (int i = i0 + tid; i < i1; i += kScoreThreads) a.units[(size_t)gi * a.max_sub + i] = su[i - i0];
  }
  // block max over present sub-blocks; -inf for blocks not yet created
  if (!VARIANT) {
    for (int jj = tid; jj < a.chunk / spb; jj += kScoreThreads) {
      const int j = i0 / spb + jj;
      if (j >= a.max_blocks) break;
      float m = -INFINITY;
      if (j < N) {
        const int e = min((j + 1) * spb, M);
        for (int i = j * spb; i < e; ++i) m = fmaxf(m, su[i - i0]);
      }
      a.block_scores[(size_t)gi * a.max_blocks + j] = m;
    }
  }
  if (!FUSED) return;

  // last chunk of this group to finish runs the query-aware selection
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.counters[gi], 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (VARIANT) variant_block_scores<VARIANT == 2>(a, gi, L, M, N, vred);
  const SelSmem S = sel_smem_carve(dsm, a.max_blocks);
  const int k = a.k_q + a.k_e;
  select_query(S, a.block_scores + (size_t)gi * a.max_blocks, a.ge_mask + (size_t)gi * Wmax,
               a.prev_sel + (size_t)gi * Wmax, a.sel + (size_t)gi * k, N, k, Wmax);
  if (a.e_flag) {
    // the rest of the attention order after the early part (Gamma_e's resident blocks, found
    // again from the same block table: nothing changes it before the residency plan below):
    // S(t) minus that part ascending, then -1
    const int W = (N + 31) / 32;
    const int ne = static_cast<int>(__ldcg(a.e_flag + (size_t)gi * kFlagStride + 2));
    resident_bits(S.ge, S.m2, a.host_k ? a.block_table + (size_t)gi * a.max_blocks : nullptr, W);
    for (int w = tid; w < W; w += kScoreThreads) S.m1[w] = S.sset[w] & ~S.m2[w];
    __syncthreads();
    int32_t* al = a.att_list + (size_t)gi * k;
    const int nr = sel_compact(S, S.m1, W, al + ne);
    for (int i = ne + nr + tid; i < k; i += kScoreThreads) al[i] = -1;
  }
  if (a.host_k) {
    PlanArgs p;
    p.block_table = a.block_table + (size_t)gi * a.max_blocks;
    p.slot_owner = a.slot_owner + (size_t)gi * a.slots;
    p.last_used = a.last_used + (size_t)gi * a.max_blocks;
    p.copy_list = a.copy_list + (size_t)gi * a.copy_stride;
    p.copy_count = a.copy_count + gi;
    p.miss_count = a.miss_count ? a.miss_count + gi : nullptr;
    p.err = a.err;
    p.L = L;
    p.bs = a.bs;
    p.slots = a.slots;
    p.page_base = gi * a.slots;
    p.max_blocks = a.max_blocks;
    plan_group(S, p);
  } else if (a.miss_count && tid == 0) {
    a.miss_count[gi] = 0;
  }
  if (tid == 0) {
    a.counters[gi] = 0u;
    a.seq_len[gi] = L;
  }
  if (a.sel_flag) {
    // everything the attention reads for this group is written: publish it
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      st_release_gpu(a.sel_flag + (size_t)gi * kFlagStride, 1u);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) append_kernel(StepArgs a) {
  const int gi = blockIdx.x;
  if (a.ready) {
    // lookahead: this group's page copies may target the tail block; they land first
    if (threadIdx.x == 0 && !wait_flag(a.ready + (size_t)gi * kFlagStride, globaltimer() + a.wait_ns))
      set_err(a.err, NOSA_ERR_TIMEOUT);
    __syncthreads();
  }
  const int len0 = a.seq_len[gi];
  if (len0 >= a.max_blocks * a.bs) {
    if (threadIdx.x == 0) set_err(a.err, NOSA_ERR_FULL);
    return;
  }
  append_token<D>(a, gi, len0);
  __syncthreads();
  if (threadIdx.x == 0) a.seq_len[gi] = len0 + 1;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(StepArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  const int gi = blockIdx.x;
  const int L = a.seq_len[gi];
  const int N = (L + a.bs - 1) / a.bs;
  const SelSmem S = sel_smem_carve(dsm, a.max_blocks);
  const int Wmax = (a.max_blocks + 31) / 32;
  const int k = a.k_q + a.k_e;
  select_evict(S, a.evict + (size_t)gi * a.max_blocks, a.prev_sel + (size_t)gi * Wmax,
               a.alive + (size_t)gi * Wmax, nullptr, N, a.k_e, Wmax);
  select_query(S, a.block_scores + (size_t)gi * a.max_blocks, nullptr, a.prev_sel + (size_t)gi * Wmax,
               a.sel + (size_t)gi * k, N, k, Wmax);
}

__global__ void __launch_bounds__(kSelThreads) plan_kernel(StepArgs a) {
  extern __shared__ __align__(16) uint8_t dsm[];
  const int gi = blockIdx.x;
  const int L = a.seq_len[gi];
  const int N = (L + a.bs - 1) / a.bs;
  const SelSmem S = sel_smem_carve(dsm, a.max_blocks);
  const int Wmax = (a.max_blocks + 31) / 32;
  const int k = a.k_q + a.k_e;
  sset_from_list(S, a.sel + (size_t)gi * k, k, N, Wmax, a.err);
  PlanArgs p;
  p.block_table = a.block_table + (size_t)gi * a.max_blocks;
  p.slot_owner = a.slot_owner + (size_t)gi * a.slots;
  p.last_used = a.last_used + (size_t)gi * a.max_blocks;
  p.copy_list = a.copy_list + (size_t)gi * a.copy_stride;
  p.copy_count = a.copy_count + gi;
  p.miss_count = a.miss_count ? a.miss_count + gi : nullptr;
  p.err = a.err;
  p.L = L;
  p.bs = a.bs;
  p.slots = a.slots;
  p.page_base = gi * a.slots;
  p.max_blocks = a.max_blocks;
  plan_group(S, p);
}

// Host -> HBM page copies over UVA (pinned host memory read by the kernel with 16-byte
// loads; NOSA's "Comunicacion de Alto Ancho de Banda"). copy_kernel: grid = (groups, CTAs per
// group), after the whole previous grid; copy_seq_kernel below: the flag-driven form.
struct CopyArgs {
  const int2* copy_list;
  int copy_stride;
  const int32_t* copy_count;
  const uint4* host_k;
  const uint4* host_v;
  uint4* k_pool;
  uint4* v_pool;
  int max_blocks, page_vec;
  uint32_t* sel_flag;    // [groups * kFlagStride] plan published (copy_seq_kernel)
  uint32_t* copy_cnt;    // [groups] CTAs done with the group (copy_seq_kernel; starts, ends at 0)
  uint32_t* copy_flag;   // [groups * kFlagStride] pages in place (copy_seq_kernel)
  uint32_t* err;
  unsigned long long wait_ns;  // limit of the bounded waits on the plan flags
};

__global__ void __launch_bounds__(256) copy_kernel(CopyArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  const int gi = blockIdx.x;
  const int n = __ldcg(a.copy_count + gi);
  for (int i = blockIdx.y; i < n; i += gridDim.y) {
    const int2 e = __ldcg(a.copy_list + (size_t)gi * a.copy_stride + i);
    const size_t src = ((size_t)gi * a.max_blocks + e.x) * a.page_vec;
    const size_t dst = (size_t)e.y * a.page_vec;
    for (int v0 = threadIdx.x; v0 < a.page_vec; v0 += 4 * blockDim.x) {
      uint4 rk[4], rv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * blockDim.x;
        if (v < a.page_vec) {
          rk[u] = a.host_k[src + v];
          rv[u] = a.host_v[src + v];
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * blockDim.x;
        if (v < a.page_vec) {
          a.k_pool[dst + v] = rk[u];
          a.v_pool[dst + v] = rv[u];
        }
      }
    }
  }
}

// Flag-driven form of the copy: a pool of CTAs walks the groups in order and shares each
// group's pages among its CTAs (one block, K and V page, per CTA at a time). PCIe stays busy
// from the first published plan on, and the pages of group g land before those of g + 1, so
// the attention of the early groups overlaps the transfers of the later ones. The CTA that
// finishes a group last publishes copy_flag (and clears the group's sel_flag and counter).
__global__ void __launch_bounds__(256) copy_seq_kernel(CopyArgs a, int ngroups) {
  griddep_launch_dependents();
  __shared__ int s_n;
  const unsigned long long deadline = globaltimer() + a.wait_ns;
  for (int gi = 0; gi < ngroups; ++gi) {
    if (threadIdx.x == 0) {
      if (!wait_flag(a.sel_flag + (size_t)gi * kFlagStride, deadline)) set_err(a.err, NOSA_ERR_TIMEOUT);
      s_n = __ldcg(a.copy_count + gi);
    }
    __syncthreads();
    const int n = s_n;
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
      const int2 e = __ldcg(a.copy_list + (size_t)gi * a.copy_stride + i);
      const size_t src = ((size_t)gi * a.max_blocks + e.x) * a.page_vec;
      const size_t dst = (size_t)e.y * a.page_vec;
      for (int v0 = threadIdx.x; v0 < a.page_vec; v0 += 4 * blockDim.x) {
        uint4 rk[4], rv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * blockDim.x;
          if (v < a.page_vec) {
            rk[u] = a.host_k[src + v];
            rv[u] = a.host_v[src + v];
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * blockDim.x;
          if (v < a.page_vec) {
            a.k_pool[dst + v] = rk[u];
            a.v_pool[dst + v] = rv[u];
          }
        }
      }
    }
    __syncthreads();  // s_n is rewritten for the next group only after every thread read it
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(a.copy_cnt + gi, 1u) == gridDim.x - 1) {
        a.copy_cnt[gi] = 0u;
        a.sel_flag[(size_t)gi * kFlagStride] = 0u;
        __threadfence();
        st_release_gpu(a.copy_flag + (size_t)gi * kFlagStride, 1u);
      }
    }
  }
}

// ------------------------------------------------------------------ state init
struct InitArgs {
  const int32_t* prefill_len;
  const uint8_t* resident;
  int32_t* seq_len;
  uint32_t* prev_sel;
  uint32_t* alive;
  int32_t* last_used;
  int32_t* block_table;
  int32_t* slot_owner;
  int2* copy_list;
  int copy_stride;
  int32_t* copy_count;
  uint32_t* err;
  int Hkv, bs, max_blocks, slots, host;
};

__global__ void __launch_bounds__(256) init_tables_kernel(InitArgs a) {
  __shared__ int red[33];
  const int gi = blockIdx.x, tid = threadIdx.x;
  const int T = a.prefill_len[gi / a.Hkv];
  const int n0 = (T + a.bs - 1) / a.bs;
  const int Wmax = (a.max_blocks + 31) / 32;
  if (tid == 0) a.seq_len[gi] = T;
  for (int w = tid; w < Wmax; w += blockDim.x) {
    a.prev_sel[(size_t)gi * Wmax + w] = word_valid_mask(w, n0);
    a.alive[(size_t)gi * Wmax + w] = word_valid_mask(w, a.max_blocks);
  }
  for (int j = tid; j < a.max_blocks; j += blockDim.x) a.last_used[(size_t)gi * a.max_blocks + j] = 0;
  int32_t* bt = a.block_table + (size_t)gi * a.max_blocks;
  int32_t* so = a.slot_owner + (size_t)gi * a.slots;
  if (!a.host) {
    for (int j = tid; j < a.max_blocks; j += blockDim.x) {
      bt[j] = gi * a.slots + j;
      so[j] = j;
    }
    if (tid == 0) a.copy_count[gi] = 0;
    return;
  }
  // resident blocks take slots 0, 1, ... in ascending block order
  const uint8_t* rf = a.resident ? a.resident + (size_t)gi * a.max_blocks : nullptr;
  uint32_t m = 0;
  if (tid < Wmax && rf) {
    for (int b = 0; b < 32; ++b) {
      const int j = tid * 32 + b;
      if (j < a.max_blocks && rf[j]) m |= 1u << b;
    }
  }
  int total;
  const int before = block_exclusive_scan(__popc(m), red, &total);
  if (total > a.slots && tid == 0) set_err(a.err, NOSA_ERR_INIT);
  for (int j = tid; j < a.max_blocks; j += blockDim.x) bt[j] = -1;
  for (int z = tid; z < a.slots; z += blockDim.x) so[z] = -1;
  __syncthreads();
  if (tid < Wmax) {
    uint32_t t = m;
    int r = before;
    while (t) {
      const int b = __ffs(t) - 1;
      t &= t - 1;
      if (r < a.slots) {
        const int j = tid * 32 + b;
        bt[j] = gi * a.slots + r;
        so[r] = j;
        a.copy_list[(size_t)gi * a.copy_stride + r] = make_int2(j, gi * a.slots + r);
      }
      ++r;
    }
  }
  if (tid == 0) a.copy_count[gi] = total < a.slots ? total : a.slots;
}

// kc[i] = mean of the present tokens of sub-block i (prefill; fp32, or rounded to bf16 with
// KC16), zero past the prefill.
template <int D, bool KC16>
__global__ void __launch_bounds__(256) init_kc_kernel(const int32_t* prefill_len, int Hkv,
                                                      const uint16_t* src, int src_pages_per_group,
                                                      float* kc, int max_sub, int bs, int s) {
  const int gi = blockIdx.y;
  const int T = prefill_len[gi / Hkv];
  constexpr int SUBS = 256 / D * 4;  // sub-blocks per CTA pass
  for (int e = threadIdx.x; e < SUBS * D; e += blockDim.x) {
    const int i = blockIdx.x * SUBS + e / D, x = e % D;
    if (i >= max_sub) continue;
    const int t0 = i * s, t1 = min(t0 + s, T);
    float sum = 0.f;
    for (int tau = t0; tau < t1; ++tau) {
      const int j = tau / bs, r = tau % bs;
      sum += bf16_bits_to_f32(src[(((size_t)gi * src_pages_per_group + j) * bs + r) * D + x]);
    }
    const float mean = (t1 > t0) ? __fdiv_rn(sum, (float)(t1 - t0)) : 0.f;
    const size_t ki = ((size_t)gi * max_sub + i) * D + x;
    if (KC16) reinterpret_cast<__nv_bfloat16*>(kc)[ki] = __float2bfloat16_rn(mean);
    else kc[ki] = mean;
  }
}

}  // namespace nosa
