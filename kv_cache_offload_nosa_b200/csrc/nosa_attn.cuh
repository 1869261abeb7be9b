// Split-K flash-decoding over the selected blocks of every GQA group.
//
// Work decomposition ("stream-K" over selected blocks): the B*Hkv*k (group,
// selected-block) tasks are laid out group after group and cut into equal
// contiguous ranges of W tasks, one range per CTA, so every CTA streams the
// same number of KV pages whatever the group boundaries. A CTA range covers
// parts of at most a few groups; for each part it writes one online-softmax
// partial (m, l, acc) per query head, and the last CTA to finish a group
// (atomic ticket, no spinning) merges the group's partials into the output.
// The (m, l, acc) state and its merge are the ones S2O's two-pass kernel
// caches (gist.science/it/paper/2602.22575, "Implementazione del Kernel").
//
// Inside a CTA: one producer warp issues TMA tile loads (128-byte swizzle, no
// multicast) of the K and V page of each task into a ring of shared-memory
// stages; BS/16 consumer warps each own 16 tokens of every page. Those 16
// tokens are the M side of both m16n8k16 bf16 products (K . q^T, then
// V^T . P^T), the group's query heads the 8 N columns: a group supplies only
// G <= 8 query rows, so with the tokens on M no row of a tile is padding. P is
// split into bf16 high + low parts (a single bf16 P would cost ~1e-3 relative
// error); with G <= 4 each head takes two columns, one per part, so a single
// product accumulates both, and the parts are summed when the partial is
// written.
#pragma once

#include "nosa_common.cuh"

namespace nosa {

constexpr int kMaxStages = 8;

struct AttnArgs {
  const uint16_t* q;          // [B][Hq][D]
  const int32_t* sel;         // [B*Hkv][k]
  const int32_t* seq_len;     // [B*Hkv]
  const int32_t* block_table; // [B*Hkv][max_blocks]
  float* out;                 // [B][Hq][D]
  float* partials;            // [B*Hkv][kPartialSlots][G][D+2]
  uint32_t* counters;         // [B*Hkv]
  uint32_t* err;
  int Hq, Hkv, G, k, max_blocks;
  int W;                      // tasks per CTA
  int total;                  // B*Hkv*k
  int stages;
  long long total_pages;
  float scale_log2;           // sigma * log2(e)
  uint32_t* sel_flag;         // [B*Hkv * kFlagStride] per-group "ready" flags, or NULL
  // early start (with sel_flag): the task order and the early flags the score kernel
  // publishes (Gamma_e first, then Gamma_q; see StepArgs), or NULL to read sel and seq_len
  const int32_t* att_list;    // [B*Hkv][k]
  uint32_t* e_flag;           // [B*Hkv * kFlagStride]: [0] flag, [1] L, [2] |Gamma_e|
  int identity;               // no host pools: block j of group g is page g * max_blocks + j
                              // (the state's block table is that identity), so no lookup
  unsigned long long wait_ns; // limit of every bounded wait, from the kernel's start
};

struct TaskInfo {
  int gi, j, L, last;         // gi < 0: no more tasks
  int seg, nseg;              // the task's partial slot in its group, and the group's slot count
};

template <int D, int BS>
struct AttnShape {
  static constexpr int NC = BS / 16;                  // consumer warps
  static constexpr int THREADS = (NC + 1) * 32;
  static constexpr int HALVES = D / 64;               // 64-column (128-byte) TMA boxes
  static constexpr int TILE = BS * 128;               // bytes of one [BS][64] box
  static constexpr int KV = BS * D * 2;               // bytes of one K (or V) page
  static constexpr int STAGE = 2 * KV;
  static size_t smem_bytes(int stages) {
    return 1024 + (size_t)stages * STAGE + 2 * kMaxStages * 8 + kMaxStages * sizeof(TaskInfo) + 64;
  }
};

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Byte offset of (row, col) in a stage operand made of HALVES swizzled [BS][64] boxes.
template <int BS>
__device__ __forceinline__ uint32_t swz(int row, int col) {
  const int h = col >> 6, chunk = (col & 63) >> 3;
  return static_cast<uint32_t>(h * BS * 128 + row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D, int BS>
// (3 CTAs per SM for register allocation: 136 registers or fewer at 64-token blocks, so one
// attention CTA fits beside two score CTAs while the step's score kernel still runs)
__global__ void __launch_bounds__(AttnShape<D, BS>::THREADS, BS == 128 ? 1 : 3)
    attn_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                AttnArgs a) {
  using SH = AttnShape<D, BS>;
  constexpr int NC = SH::NC;
  constexpr int MT = D / 16;    // 16-dim m-tiles of the output (O^T)
  constexpr int KS = D / 16;    // 16-wide k-steps of K.Qc
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int ST = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)ST * SH::STAGE);
  uint64_t* empty = full + kMaxStages;
  TaskInfo* info = reinterpret_cast<TaskInfo*>(empty + kMaxStages);
  int* s_flag = reinterpret_cast<int*>(info + kMaxStages);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int task0 = blockIdx.x * a.W;
  const int ntask = min(a.W, a.total - task0);
  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NC);
    }
    fence_barrier_init();
  }
  if (warp == NC && lane == 0) {
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  __syncthreads();
  // sel, seq_len, the block table and the appended token come from the previous kernel:
  // either wait for that whole grid, or (flags) for the one group a task belongs to
  const bool flags = a.sel_flag != nullptr;
  if (!flags) griddep_wait();
  const unsigned long long deadline = globaltimer() + a.wait_ns;

  if (warp == NC) {
    // ---------------------------------------------------------------- producer
    // The CTA's W tasks are cut at group boundaries into ranges, each ending in a partial
    // (m, l, acc) slot of its group. A range is taken in parts that wait for the same flag:
    // with early publication a group's first |Gamma_e| positions (its query-agnostic blocks,
    // with the context length) are ready before the query-aware selection, the rest once the
    // whole selection (and, with host pools, its page copies) is in place. Per part the warp
    // resolves 32 tasks' metadata at once (block -> page, in parallel across lanes); lane 0
    // then issues the tile loads in task order. Lane 0 acquires each flag; the warp barrier
    // orders the other lanes' loads (L2, __ldcg) after that acquire.
    const bool early = a.att_list != nullptr;
    const int32_t* list = early ? a.att_list : a.sel;
    int it = 0;  // tasks issued (stage ring position)
    bool abort = false;
    for (int sr = 0; sr < ntask && !abort;) {
      // the group, the positions [pa, pb) of its order in this CTA, and the partial slot
      const int gi = (task0 + sr) / a.k;
      const int pa = task0 + sr - gi * a.k;
      const int pb = min(task0 + ntask, (gi + 1) * a.k) - gi * a.k;
      const int first = (int)(((long long)gi * a.k) / a.W);
      const int lastc = (int)(((long long)gi * a.k + a.k - 1) / a.W);
      const int seg = blockIdx.x - first, nseg = lastc - first + 1;
      sr += pb - pa;
      const int tbase = gi * a.k;  // task index of the group's position 0
      for (int p = pa; p < pb && !abort;) {
        int pend = pb, L;
        const uint32_t* f = flags ? a.sel_flag + (size_t)gi * kFlagStride : nullptr;
        if (early) {
          const uint32_t* ef = a.e_flag + (size_t)gi * kFlagStride;
          if (lane == 0 && !wait_flag(ef, deadline)) set_err(a.err, NOSA_ERR_TIMEOUT);
          __syncwarp();
          L = static_cast<int>(__ldcg(ef + 1));
          const int ne = static_cast<int>(__ldcg(ef + 2));
          if (p < ne) {  // query-agnostic part: ready now
            pend = min(pb, ne);
            f = nullptr;
          }
        }
        if (f) {
          if (lane == 0 && !wait_flag(f, deadline)) set_err(a.err, NOSA_ERR_TIMEOUT);
          __syncwarp();
        }
        if (!early) L = __ldcg(a.seq_len + gi);
        if (flags && lane == 0) fence_proxy_async_global();  // pages written before the flags
        const int N = (L + BS - 1) / BS;
        for (int base = p; base < pend && !abort; base += 32) {
          const int p_l = base + lane;
          int j_l = -1, page_l = -1;
          if (p_l < pend) {
            j_l = __ldcg(list + tbase + p_l);
            if (j_l >= N) {
              set_err(a.err, NOSA_ERR_SEL);
              j_l = -1;
            }
            if (j_l >= 0) {
              page_l = a.identity ? gi * a.max_blocks + j_l
                                  : __ldcg(a.block_table + (size_t)gi * a.max_blocks + j_l);
              if (page_l < 0 || page_l >= a.total_pages) {
                set_err(a.err, NOSA_ERR_BLOCK_TABLE);
                j_l = -1;
              }
            }
          }
          const int nb = min(32, pend - base);
          __syncwarp();
          for (int v = 0; v < nb; ++v) {
            const int j = __shfl_sync(0xffffffffu, j_l, v);
            const int page = __shfl_sync(0xffffffffu, page_l, v);
            if (lane == 0) {
              const int s = it % ST, round = it / ST;
              if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, deadline)) {
                set_err(a.err, NOSA_ERR_TIMEOUT);
                abort = true;
              } else {
                TaskInfo ti;
                ti.gi = gi;
                ti.j = j;
                ti.L = L;
                ti.last = (base + v == pb - 1);
                ti.seg = seg;
                ti.nseg = nseg;
                info[s] = ti;
                if (j >= 0) {
                  mbar_arrive_expect_tx(&full[s], SH::STAGE);
                  uint8_t* st = smem + (size_t)s * SH::STAGE;
#pragma unroll
                  for (int h = 0; h < SH::HALVES; ++h) {
                    tma_load_2d(st + h * SH::TILE, &tmk, &full[s], 64 * h, page * BS);
                    tma_load_2d(st + SH::KV + h * SH::TILE, &tmv, &full[s], 64 * h, page * BS);
                  }
                } else {
                  mbar_arrive(&full[s]);
                }
                ++it;
              }
            }
            abort = __shfl_sync(0xffffffffu, abort, 0);
            if (abort) break;
          }
        }
        p = pend;
      }
    }
    // end of the CTA's tasks: a task with gi < 0 stops the consumers
    if (lane == 0 && !abort) {
      const int s = it % ST, round = it / ST;
      if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, deadline)) {
        set_err(a.err, NOSA_ERR_TIMEOUT);
      } else {
        TaskInfo ti;
        ti.gi = -1;
        ti.j = -1;
        ti.L = 0;
        ti.last = 0;
        ti.seg = 0;
        ti.nseg = 0;
        info[s] = ti;
        mbar_arrive(&full[s]);
        ++it;
      }
    }
    const int issued = it;
    // never leave the CTA with a tile load in flight
    if (lane == 0)
      for (int i = max(0, issued - ST); i < issued; ++i)
        mbar_wait(&full[i % ST], (i / ST) & 1, deadline);
    return;
  }

  // ---------------------------------------------------------------- consumers
  // Per warp, the 16 tokens it owns in every page are the M rows of both products:
  //   S^T  = K . Qc      A: K rows straight from shared memory (ldmatrix),
  //                      B: Qc, the group's query heads as 8 columns;
  //   O^T += V^T . P^T   A: V rows through ldmatrix.trans,
  //                      B: P^T, put in place from the S^T accumulator layout by movmatrix.trans.
  // With G <= 4 every head fills two columns, h and h + 4: column h carries the high bf16 part
  // of P and column h + 4 the low part (P - high), so one product accumulates both and the
  // halves are added when the partial is written. With G = 8 a second product adds the low parts.
  const int r = lane >> 2, c4 = lane & 3;
  const bool wide = a.G > 4;
  auto col_head = [&](int n) { return wide ? n : (n & 3); };
  const int h0 = col_head(2 * c4), h1 = col_head(2 * c4 + 1);  // heads of this lane's columns
  const bool cv0 = h0 < a.G, cv1 = h1 < a.G;
  const bool lo_cols = !wide && c4 >= 2;                       // columns 4..7: low parts
  const bool owner = !wide ? c4 < 2 : true;                    // writes its columns' results
  const int qhead = col_head(r);                               // B column r of Qc
  uint32_t qb[KS][2];
  float acc[MT][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;    // columns 2*c4 and 2*c4 + 1
  int cur = -1;

  for (int i = 0;; ++i) {
    const int s = i % ST;
    if (!mbar_wait(&full[s], (i / ST) & 1, deadline)) {
      set_err(a.err, NOSA_ERR_TIMEOUT);
      break;
    }
    const TaskInfo ti = info[s];
    if (ti.gi < 0) break;  // the producer has no more tasks (nothing in this stage to release)
    uint8_t* kst = smem + (size_t)s * SH::STAGE;
    uint8_t* vst = kst + SH::KV;
    if (ti.gi != cur) {
      cur = ti.gi;
      const int b = cur / a.Hkv, g = cur % a.Hkv;
      const bool qok = qhead < a.G;
      const uint16_t* qrow = a.q + ((size_t)b * a.Hq + g * a.G + (qok ? qhead : 0)) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qb[ks][0] = qok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c4) : 0u;
        qb[ks][1] = qok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c4) : 0u;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    }
    bool wrote_smem = false, released = false;
    const int tok0 = ti.j * BS + 16 * warp;
    const int nval = (ti.j >= 0) ? min(16, ti.L - tok0) : 0;
    if (nval > 0) {
      if (nval < 16) {
        // rows past the context may hold anything; zero them so 0 * V stays 0
        for (int e = lane; e < (16 - nval) * (D / 8); e += 32) {
          const int row = 16 * warp + nval + e / (D / 8), col = 8 * (e % (D / 8));
          *reinterpret_cast<uint4*>(vst + swz<BS>(row, col)) = make_uint4(0, 0, 0, 0);
        }
        wrote_smem = true;
        __syncwarp();
      }
      // S^T for 16 tokens x 8 columns; two accumulators halve the dependent mma chain
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int mi = lane >> 3, r8 = lane & 7;
        const int row = 16 * warp + 8 * (mi & 1) + r8;
        const uint32_t kbase = smem_u32(kst);
#pragma unroll
        for (int ks = 0; ks < KS; ks += 2) {
          uint32_t x0, x1, x2, x3, y0, y1, y2, y3;
          ldsm_x4(kbase + swz<BS>(row, 16 * ks + 8 * (mi >> 1)), x0, x1, x2, x3);
          ldsm_x4(kbase + swz<BS>(row, 16 * ks + 16 + 8 * (mi >> 1)), y0, y1, y2, y3);
          mma_16816(sa, x0, x1, x2, x3, qb[ks][0], qb[ks][1]);
          mma_16816(sb, y0, y1, y2, y3, qb[ks + 1][0], qb[ks + 1][1]);
        }
      }
      // online softmax (log2 domain) per column; this lane: tokens r and r + 8
      const bool t0 = r < nval, t1 = r + 8 < nval;
      const float x0 = (cv0 && t0) ? (sa[0] + sb[0]) * a.scale_log2 : -INFINITY;
      const float x1 = (cv1 && t0) ? (sa[1] + sb[1]) * a.scale_log2 : -INFINITY;
      const float x2 = (cv0 && t1) ? (sa[2] + sb[2]) * a.scale_log2 : -INFINITY;
      const float x3 = (cv1 && t1) ? (sa[3] + sb[3]) * a.scale_log2 : -INFINITY;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0, mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
      const float al0 = (mn0 != m0) ? ex2(m0 - mu0) : 1.f;
      const float al1 = (mn1 != m1) ? ex2(m1 - mu1) : 1.f;
      const float p0 = ex2(x0 - mu0), p2 = ex2(x2 - mu0);
      const float p1 = ex2(x1 - mu1), p3 = ex2(x3 - mu1);
      l0 = l0 * al0 + (p0 + p2);
      l1 = l1 * al1 + (p1 + p3);
      // the running max of most columns stops moving after the first blocks: rescale only
      // when some column's max changed (alpha == 1 exactly otherwise)
      const bool moved = (mn0 != m0) || (mn1 != m1);
      m0 = mn0;
      m1 = mn1;
      if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          acc[mt][0] *= al0;
          acc[mt][1] *= al1;
          acc[mt][2] *= al0;
          acc[mt][3] *= al1;
        }
      }
      // P as bf16 high + low parts, in the S^T layout (rows = tokens r / r + 8)
      const uint32_t hi01 = pack_bf16(p0, p1), hi23 = pack_bf16(p2, p3);
      const __nv_bfloat162 e01 = *reinterpret_cast<const __nv_bfloat162*>(&hi01);
      const __nv_bfloat162 e23 = *reinterpret_cast<const __nv_bfloat162*>(&hi23);
      const uint32_t lo01 = pack_bf16(p0 - __low2float(e01), p1 - __high2float(e01));
      const uint32_t lo23 = pack_bf16(p2 - __low2float(e23), p3 - __high2float(e23));
      // P^T as the B operand: column n = lane >> 2, tokens 2*c4.. (b0) and 8 + 2*c4.. (b1)
      const uint32_t pb0 = movmatrix_t(lo_cols ? lo01 : hi01);
      const uint32_t pb1 = movmatrix_t(lo_cols ? lo23 : hi23);
      uint32_t pl0 = 0u, pl1 = 0u;
      if (wide) {
        pl0 = movmatrix_t(lo01);
        pl1 = movmatrix_t(lo23);
      }
      {
        const int mi = lane >> 3, r8 = lane & 7;
        const int row = 16 * warp + 8 * (mi >> 1) + r8;
        const uint32_t vbase = smem_u32(vst);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          uint32_t v0, v1, v2, v3;
          ldsm_x4_t(vbase + swz<BS>(row, 16 * mt + 8 * (mi & 1)), v0, v1, v2, v3);
          mma_16816(acc[mt], v0, v1, v2, v3, pb0, pb1);
          if (wide) mma_16816(acc[mt], v0, v1, v2, v3, pl0, pl1);
        }
      }
    }

    if (ti.last) {
      // ------------------------------------------------ flush this group's part
      named_bar(1, NC * 32);  // every consumer is done reading stage s
      float L0 = l0, L1 = l1;  // sums over the warp's 16 token rows
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        L0 += __shfl_xor_sync(0xffffffffu, L0, o);
        L1 += __shfl_xor_sync(0xffffffffu, L1, o);
      }
      if (!wide) {
        // high part (columns 0..3, lanes c4 < 2) + low part (columns 4..7, lanes c4 + 2)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[mt][e] += __shfl_xor_sync(0xffffffffu, acc[mt][e], 2);
      }
      float* scr = reinterpret_cast<float*>(kst);  // [NC][G][D+2] in the spent stage
      if (owner) {
        float* w0 = scr + ((size_t)warp * a.G + h0) * (D + 2);
        float* w1 = scr + ((size_t)warp * a.G + h1) * (D + 2);
        if (r == 0) {
          if (cv0) {
            w0[0] = m0;
            w0[1] = L0;
          }
          if (cv1) {
            w1[0] = m1;
            w1[1] = L1;
          }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          if (cv0) {
            w0[2 + 16 * mt + r] = acc[mt][0];
            w0[2 + 16 * mt + 8 + r] = acc[mt][2];
          }
          if (cv1) {
            w1[2 + 16 * mt + r] = acc[mt][1];
            w1[2 + 16 * mt + 8 + r] = acc[mt][3];
          }
        }
      }
      wrote_smem = true;
      named_bar(1, NC * 32);
      const int gi = ti.gi;
      const int nseg = ti.nseg, seg = ti.seg;
      const int GE = a.G * (D + 2);
      float* part = a.partials + ((size_t)gi * kPartialSlots + seg) * GE;
      for (int e = tid; e < GE; e += NC * 32) {
        const int h = e / (D + 2), col = e % (D + 2);
        float M = -INFINITY;
        for (int w = 0; w < NC; ++w) M = fmaxf(M, scr[((size_t)w * a.G + h) * (D + 2)]);
        float v;
        if (col == 0) {
          v = M;
        } else {
          v = 0.f;
          if (M != -INFINITY)
            for (int w = 0; w < NC; ++w) {
              const float* ww = scr + ((size_t)w * a.G + h) * (D + 2);
              v += ww[col] * exp2f(ww[0] - M);
            }
        }
        part[e] = v;
      }
      // the scratch in stage s has been read by everyone: hand the stage back to the producer
      // now, so the ticket and the combine below overlap the next tiles' loads
      named_bar(1, NC * 32);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      released = true;
      __threadfence();
      named_bar(1, NC * 32);
      if (tid == 0) *s_flag = (atomicAdd(&a.counters[gi], 1u) == (unsigned)(nseg - 1));
      named_bar(1, NC * 32);
      if (*s_flag) {
        __threadfence();
        const float* p0 = a.partials + (size_t)gi * kPartialSlots * GE;
        const int b = gi / a.Hkv, g = gi % a.Hkv;
        for (int e = tid; e < a.G * D; e += NC * 32) {
          const int h = e / D, col = e % D;
          float M = -INFINITY;
          for (int sg = 0; sg < nseg; ++sg) M = fmaxf(M, __ldcg(p0 + (size_t)sg * GE + h * (D + 2)));
          float num = 0.f, den = 0.f;
          if (M != -INFINITY)
            for (int sg = 0; sg < nseg; ++sg) {
              const float* ps = p0 + (size_t)sg * GE + h * (D + 2);
              const float f = exp2f(__ldcg(ps) - M);
              den += __ldcg(ps + 1) * f;
              num += __ldcg(ps + 2 + col) * f;
            }
          a.out[((size_t)b * a.Hq + g * a.G + h) * D + col] = (den > 0.f) ? num / den : 0.f;
        }
        if (tid == 0) {
          a.counters[gi] = 0u;
          if (flags) a.sel_flag[(size_t)gi * kFlagStride] = 0u;  // every CTA of the group passed its wait
          if (a.e_flag) {
            a.e_flag[(size_t)gi * kFlagStride] = 0u;
            a.e_flag[(size_t)gi * kFlagStride + 3] = 0u;
          }
        }
      }
      named_bar(1, NC * 32);
      // the partial is written: the next task starts a new one
      cur = -1;
    }
    if (!released) {
      if (wrote_smem) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
}

}  // namespace nosa
