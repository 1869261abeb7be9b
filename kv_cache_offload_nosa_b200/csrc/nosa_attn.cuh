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
// stages; BS/16 consumer warps each own 16 tokens of every page. Per warp the
// G query heads are rows 0..G-1 of an m16n8k16 bf16 mma (other rows zero);
// q.K^T uses K straight from shared memory (ldmatrix). P.V uses V through
// ldmatrix.trans with P split into bf16 hi + lo parts (a single bf16 P would
// cost ~1e-3 relative error): rows 0..7 of the A operand carry P_hi and rows
// 8..15 carry P_lo, so one mma accumulates both and the two halves of the
// accumulator are summed when the partial is written.
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
  int identity;               // no host pools: block j of group g is page g * max_blocks + j
                              // (the state's block table is that identity), so no lookup
  unsigned long long wait_ns; // limit of every bounded wait, from the kernel's start
};

struct TaskInfo {
  int gi, j, L, last;
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
__global__ void __launch_bounds__(AttnShape<D, BS>::THREADS, BS == 128 ? 1 : 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                AttnArgs a) {
  using SH = AttnShape<D, BS>;
  constexpr int NC = SH::NC;
  constexpr int NT = D / 8;     // 8-column n-tiles of the output
  constexpr int KS = D / 16;    // 16-wide k-steps of q.K^T
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
    // The warp resolves 32 tasks' metadata at once (sel -> block table, in parallel
    // across lanes); lane 0 then issues the tile loads in task order.
    int issued = 0;
    bool abort = false;
    for (int base = 0; base < ntask && !abort; base += 32) {
      const int i_l = base + lane;
      int gi_l = 0, j_l = -1, L_l = 0, page_l = -1;
      if (flags) {
        // lane 0 acquires the flags of the batch's groups (contiguous, in order); the warp
        // barrier orders the other lanes' loads below (L2, __ldcg) after those acquires
        if (lane == 0) {
          const int g1 = (task0 + min(base + 32, ntask) - 1) / a.k;
          for (int g = (task0 + base) / a.k; g <= g1; ++g)
            if (!wait_flag(a.sel_flag + (size_t)g * kFlagStride, deadline)) set_err(a.err, NOSA_ERR_TIMEOUT);
        }
        __syncwarp();
      }
      if (i_l < ntask) {
        const int t = task0 + i_l;
        gi_l = t / a.k;
        L_l = __ldcg(a.seq_len + gi_l);
        const int N = (L_l + BS - 1) / BS;
        j_l = __ldcg(a.sel + t);
        if (j_l >= N) {
          set_err(a.err, NOSA_ERR_SEL);
          j_l = -1;
        }
        if (j_l >= 0) {
          page_l = a.identity ? gi_l * a.max_blocks + j_l
                              : __ldcg(a.block_table + (size_t)gi_l * a.max_blocks + j_l);
          if (page_l < 0 || page_l >= a.total_pages) {
            set_err(a.err, NOSA_ERR_BLOCK_TABLE);
            j_l = -1;
          }
        }
      }
      const int nb = min(32, ntask - base);
      __syncwarp();
      if (flags && lane == 0) fence_proxy_async_global();  // pages written before the flags
      for (int u = 0; u < nb; ++u) {
        const int gi = __shfl_sync(0xffffffffu, gi_l, u);
        const int j = __shfl_sync(0xffffffffu, j_l, u);
        const int L = __shfl_sync(0xffffffffu, L_l, u);
        const int page = __shfl_sync(0xffffffffu, page_l, u);
        const int i = base + u;
        if (lane == 0) {
          const int s = i % ST, round = i / ST;
          if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, deadline)) {
            set_err(a.err, NOSA_ERR_TIMEOUT);
            abort = true;
          } else {
            TaskInfo ti;
            ti.gi = gi;
            ti.j = j;
            ti.L = L;
            ti.last = (i == ntask - 1) || ((task0 + i + 1) / a.k != gi);
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
            issued = i + 1;
          }
        }
        abort = __shfl_sync(0xffffffffu, abort, 0);
        if (abort) break;
      }
    }
    // never leave the CTA with a tile load in flight
    if (lane == 0)
      for (int i = max(0, issued - ST); i < issued; ++i)
        mbar_wait(&full[i % ST], (i / ST) & 1, deadline);
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int hrow = lane >> 2, c4 = lane & 3;
  const bool row_ok = hrow < a.G;
  uint32_t qa[KS][2];
  float acc[NT][4];
  float m_run = -INFINITY, l_run = 0.f;
  int cur = -1;

  for (int i = 0; i < ntask; ++i) {
    const int s = i % ST;
    if (!mbar_wait(&full[s], (i / ST) & 1, deadline)) {
      set_err(a.err, NOSA_ERR_TIMEOUT);
      break;
    }
    const TaskInfo ti = info[s];
    uint8_t* kst = smem + (size_t)s * SH::STAGE;
    uint8_t* vst = kst + SH::KV;
    if (ti.gi != cur) {
      cur = ti.gi;
      const int b = cur / a.Hkv, g = cur % a.Hkv;
      const uint16_t* qrow = a.q + ((size_t)b * a.Hq + g * a.G + hrow) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qa[ks][0] = row_ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c4) : 0u;
        qa[ks][1] = row_ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c4) : 0u;
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
      m_run = -INFINITY;
      l_run = 0.f;
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
      // S = Q K^T for 16 tokens: two n-tiles of 8 tokens
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int mi = lane >> 3, r8 = lane & 7;
        const int row = 16 * warp + 8 * (mi >> 1) + r8;
        const uint32_t kbase = smem_u32(kst);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kbase + swz<BS>(row, 16 * ks + 8 * (mi & 1)), b0, b1, b2, b3);
          mma_16816(sc[0], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
          mma_16816(sc[1], qa[ks][0], 0u, qa[ks][1], 0u, b2, b3);
        }
      }
      // online softmax (log2 domain); row hrow, tokens 8*nt + 2*c4 + e
      float p[2][2];
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tk = 8 * nt + 2 * c4 + e;
          const float v = (row_ok && tk < nval) ? sc[nt][e] * a.scale_log2 : -INFINITY;
          p[nt][e] = v;
          mx = fmaxf(mx, v);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m_new != m_run) ? ex2(m_run - m_use) : 1.f;
      float psum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          p[nt][e] = ex2(p[nt][e] - m_use);
          psum += p[nt][e];
        }
      l_run = l_run * alpha + psum;
      // the running max of most rows stops moving after the first blocks: rescale only when
      // some row's max changed (alpha == 1 exactly otherwise)
      const bool moved = m_new != m_run;
      m_run = m_new;
      if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          acc[n][0] *= alpha;
          acc[n][1] *= alpha;
          acc[n][2] *= alpha;
          acc[n][3] *= alpha;
        }
      }
      // P as bf16 hi + lo (A operand rows = heads, k = 16 tokens)
      const uint32_t ah0 = pack_bf16(p[0][0], p[0][1]);
      const uint32_t ah2 = pack_bf16(p[1][0], p[1][1]);
      const __nv_bfloat162 h0 = *reinterpret_cast<const __nv_bfloat162*>(&ah0);
      const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&ah2);
      const uint32_t al0 = pack_bf16(p[0][0] - __low2float(h0), p[0][1] - __high2float(h0));
      const uint32_t al2 = pack_bf16(p[1][0] - __low2float(h2), p[1][1] - __high2float(h2));
      {
        const int mi = lane >> 3, r8 = lane & 7;
        const int row = 16 * warp + 8 * (mi & 1) + r8;
        const uint32_t vbase = smem_u32(vst);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vbase + swz<BS>(row, 16 * np + 8 * (mi >> 1)), b0, b1, b2, b3);
          mma_16816(acc[2 * np], ah0, al0, ah2, al2, b0, b1);
          mma_16816(acc[2 * np + 1], ah0, al0, ah2, al2, b2, b3);
        }
      }
    }

    if (ti.last) {
      // ------------------------------------------------ flush this group's part
      named_bar(1, NC * 32);  // every consumer is done reading stage s
      float l = l_run;
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      float* scr = reinterpret_cast<float*>(kst);  // [NC][G][D+2] in the spent stage
      if (row_ok) {
        float* w = scr + ((size_t)warp * a.G + hrow) * (D + 2);
        if (c4 == 0) {
          w[0] = m_run;
          w[1] = l;
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          w[2 + 8 * n + 2 * c4] = acc[n][0] + acc[n][2];
          w[3 + 8 * n + 2 * c4] = acc[n][1] + acc[n][3];
        }
      }
      wrote_smem = true;
      named_bar(1, NC * 32);
      const int gi = ti.gi;
      const int first = (int)(((long long)gi * a.k) / a.W);
      const int lastc = (int)(((long long)gi * a.k + a.k - 1) / a.W);
      const int nseg = lastc - first + 1;
      const int seg = blockIdx.x - first;
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
        }
      }
      named_bar(1, NC * 32);
    }
    if (!released) {
      if (wrote_smem) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
}

}  // namespace nosa
