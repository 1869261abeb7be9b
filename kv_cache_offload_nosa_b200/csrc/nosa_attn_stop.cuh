// Attention with S2O's monotone-gain early stop over the selected blocks (S2O,
// gist.science/it/paper/2602.22575, "Regola di Arresto Anticipato"): a group's blocks are
// visited in decreasing block score (the estimated importance; ties to the lower index) and
// each query head stops after the first block whose gain in softmax mass falls below
// tau times the mass accumulated so far (that block included).
//
// The rule is sequential along the order, so one CTA handles one group: the producer warp
// streams the pages in visiting order through the same TMA ring as attn_kernel, the BS/16
// consumer warps each own 16 tokens of every page. After each block the consumers exchange
// their per-head (running max, mass, gain of the block) through shared memory and every warp
// takes the same decision; a stopped head's logits are masked to -inf from then on, so its
// state no longer changes. Once every head has stopped the producer ends the stream early.
#pragma once

#include "nosa_attn.cuh"

namespace nosa {

// Named barrier over nthreads threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

constexpr int kStopMaxK = 1024;  // selected blocks per group the early-stop kernel ranks

struct StopArgs {
  const float* scores;  // [B*Hkv][max_blocks] the step's block scores
  float tau;            // a head stops once a block's gain < tau * its mass
  int32_t* used;        // [B*Hq] blocks each head visited
};

template <int D, int BS>
struct StopShape {
  using SH = AttnShape<D, BS>;
  static constexpr int NC = SH::NC;
  // after the stages: barriers and task infos (as attn_kernel), then the order, the selected
  // entries with their scores and pages, the pages in order, the per-warp exchange and the
  // final merge
  static size_t extra_bytes(int G) {
    return 2 * kMaxStages * 8 + kMaxStages * sizeof(TaskInfo) + 5 * (size_t)kStopMaxK * 4 +
           (size_t)NC * 8 * 3 * 4 + (size_t)NC * G * (D + 2) * 4 + 64;
  }
  static size_t smem_bytes(int stages, int G) { return 1024 + (size_t)stages * SH::STAGE + extra_bytes(G); }
};

template <int D, int BS>
__global__ void __launch_bounds__(AttnShape<D, BS>::THREADS, 1)
    attn_stop_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     AttnArgs a, StopArgs x) {
  using SH = AttnShape<D, BS>;
  constexpr int NC = SH::NC;
  constexpr int NT = D / 8;
  constexpr int KS = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int ST = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)ST * SH::STAGE);
  uint64_t* empty = full + kMaxStages;
  TaskInfo* info = reinterpret_cast<TaskInfo*>(empty + kMaxStages);
  int* order = reinterpret_cast<int*>(info + kMaxStages);  // block at each visiting position
  int* ent = order + kStopMaxK;                            // selected block of each entry, or -1
  float* esc = reinterpret_cast<float*>(ent + kStopMaxK);  // its score
  int* epg = reinterpret_cast<int*>(esc + kStopMaxK);      // its page
  int* pages = epg + kStopMaxK;                            // page of each visiting position
  float* xch = reinterpret_cast<float*>(pages + kStopMaxK);  // [NC][8][3] (max, mass, gain)
  float* mrg = xch + NC * 8 * 3;                             // [NC][G][D+2] final merge
  volatile int* s_all_stopped = reinterpret_cast<volatile int*>(mrg + (size_t)NC * a.G * (D + 2));

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gi = blockIdx.x;
  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NC);
    }
    *s_all_stopped = 0;
    fence_barrier_init();
  }
  if (warp == NC && lane == 0) {
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  // sel, the block scores, seq_len and the block table come from the previous kernels: wait
  // for that whole grid, or (flags) for this group's flag, which this CTA alone waits on
  const bool flags = a.sel_flag != nullptr;
  if (!flags) griddep_wait();
  const unsigned long long deadline = globaltimer() + a.wait_ns;
  if (flags && tid == 0) {
    if (!wait_flag(a.sel_flag + (size_t)gi * kFlagStride, deadline)) set_err(a.err, NOSA_ERR_TIMEOUT);
    a.sel_flag[(size_t)gi * kFlagStride] = 0u;
  }
  __syncthreads();
  const int L = __ldcg(a.seq_len + gi);
  const int N = (L + BS - 1) / BS;
  // each selected block with its score and page (independent loads: one round trip)
  for (int w = tid; w < a.k; w += blockDim.x) {
    const int j = __ldcg(a.sel + (size_t)gi * a.k + w);
    if (j >= N) set_err(a.err, NOSA_ERR_SEL);
    const bool ok = j >= 0 && j < N;
    float sj = 0.f;
    int page = -1;
    if (ok) {
      sj = __ldcg(x.scores + (size_t)gi * a.max_blocks + j);
      page = __ldcg(a.block_table + (size_t)gi * a.max_blocks + j);
      if (page < 0 || page >= a.total_pages) {
        set_err(a.err, NOSA_ERR_BLOCK_TABLE);
        page = -1;
      }
    }
    ent[w] = ok ? j : -1;
    esc[w] = sj;
    epg[w] = page;
  }
  __syncthreads();
  // visiting order: selected blocks by decreasing score, ties to the lower index
  for (int w = tid; w < a.k; w += blockDim.x) {
    const int j = ent[w];
    if (j < 0) continue;
    const float sj = esc[w];
    int rank = 0;
    for (int w2 = 0; w2 < a.k; ++w2) {
      const int j2 = ent[w2];
      rank += (j2 >= 0) && (esc[w2] > sj || (esc[w2] == sj && j2 < j));
    }
    order[rank] = j;
    pages[rank] = epg[w];
  }
  int nvis = 0;  // selected blocks of the group
  for (int w = 0; w < a.k; ++w) nvis += (ent[w] >= 0);
  __syncthreads();

  if (warp == NC) {
    // ---------------------------------------------------------------- producer (lane 0)
    if (lane == 0) {
      int issued = 0;
      for (int p = 0;; ++p) {
        const int s = p % ST, round = p / ST;
        if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, deadline)) {
          set_err(a.err, NOSA_ERR_TIMEOUT);
          break;
        }
        TaskInfo ti;
        ti.gi = gi;
        ti.L = L;
        ti.last = 0;
        if (p >= nvis || *s_all_stopped) {
          ti.j = -2;  // end of the stream
          info[s] = ti;
          mbar_arrive(&full[s]);
          issued = p + 1;
          break;
        }
        const int page = pages[p];
        ti.j = (page >= 0) ? order[p] : -1;
        info[s] = ti;
        if (page >= 0) {
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
        issued = p + 1;
      }
      // never leave the CTA with a tile load in flight
      for (int i = max(0, issued - ST); i < issued; ++i) mbar_wait(&full[i % ST], (i / ST) & 1, deadline);
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int hrow = lane >> 2, c4 = lane & 3;
  const bool row_ok = hrow < a.G;
  const int b = gi / a.Hkv, g = gi % a.Hkv;
  uint32_t qa[KS][2];
  {
    const uint16_t* qrow = a.q + ((size_t)b * a.Hq + g * a.G + hrow) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa[ks][0] = row_ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c4) : 0u;
      qa[ks][1] = row_ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c4) : 0u;
    }
  }
  float acc[NT][4];
#pragma unroll
  for (int nn = 0; nn < NT; ++nn) acc[nn][0] = acc[nn][1] = acc[nn][2] = acc[nn][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  bool active = row_ok;   // this lane's head row still visits blocks
  int used = 0;
  bool all_stopped = false;

  for (int i = 0;; ++i) {
    const int s = i % ST;
    const bool ok = mbar_wait(&full[s], (i / ST) & 1, deadline);
    if (!ok) set_err(a.err, NOSA_ERR_TIMEOUT);
    TaskInfo ti;
    ti.j = -3;
    if (ok) ti = info[s];
    uint8_t* kst = smem + (size_t)s * SH::STAGE;
    uint8_t* vst = kst + SH::KV;
    bool wrote_smem = false;
    // the end marker (or a timed-out wait) ends the loop; every warp decides at the barrier
    // below, together, so no warp is left waiting at a later one
    const bool end = ti.j == -2 || ti.j == -3;
    const bool work = !end && ti.j >= 0 && !all_stopped;
    if (work) {
      const int tok0 = ti.j * BS + 16 * warp;
      const int nval = min(16, ti.L - tok0);
      float psum = 0.f;
      if (nval > 0) {
        if (nval < 16) {
          for (int e = lane; e < (16 - nval) * (D / 8); e += 32) {
            const int row = 16 * warp + nval + e / (D / 8), col = 8 * (e % (D / 8));
            *reinterpret_cast<uint4*>(vst + swz<BS>(row, col)) = make_uint4(0, 0, 0, 0);
          }
          wrote_smem = true;
          __syncwarp();
        }
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
        float p[2][2];
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tk = 8 * nt + 2 * c4 + e;
            const float v = (active && tk < nval) ? sc[nt][e] * a.scale_log2 : -INFINITY;
            p[nt][e] = v;
            mx = fmaxf(mx, v);
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = (m_new != m_run) ? ex2(m_run - m_use) : 1.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            p[nt][e] = ex2(p[nt][e] - m_use);
            psum += p[nt][e];
          }
        l_run = l_run * alpha + psum;
        const bool moved = m_new != m_run;
        m_run = m_new;
        if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
          for (int nn = 0; nn < NT; ++nn) {
            acc[nn][0] *= alpha;
            acc[nn][1] *= alpha;
            acc[nn][2] *= alpha;
            acc[nn][3] *= alpha;
          }
        }
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
      // this warp's share of each head row: running max, mass (block included), gain
      float lq = l_run, gq = psum;
      lq += __shfl_xor_sync(0xffffffffu, lq, 1);
      lq += __shfl_xor_sync(0xffffffffu, lq, 2);
      gq += __shfl_xor_sync(0xffffffffu, gq, 1);
      gq += __shfl_xor_sync(0xffffffffu, gq, 2);
      if (c4 == 0) {
        float* x = xch + ((size_t)warp * 8 + hrow) * 3;
        x[0] = m_run;
        x[1] = lq;
        x[2] = gq;
      }
    }
    // every warp's share of this block is in xch; leave together at the end
    if (named_bar_or(1, NC * 32, end)) {
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&empty[s]);
      break;
    }
    if (work && active) {
      float M = -INFINITY;
      for (int w = 0; w < NC; ++w) M = fmaxf(M, xch[((size_t)w * 8 + hrow) * 3]);
      float lt = 0.f, gt = 0.f;
      if (M != -INFINITY)
        for (int w = 0; w < NC; ++w) {
          const float* x = xch + ((size_t)w * 8 + hrow) * 3;
          const float f = ex2(x[0] - M);
          lt += x[1] * f;
          gt += x[2] * f;
        }
      ++used;
      if (gt < x.tau * lt) active = false;  // the head keeps this block and stops
    }
    all_stopped = !__any_sync(0xffffffffu, active);
    if (all_stopped && warp == 0 && lane == 0) *s_all_stopped = 1;
    named_bar(1, NC * 32);  // xch is rewritten only after every warp has read it
    if (wrote_smem) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // merge the warps' (m, l, acc) and write the output of every head row
  float l = l_run;
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (row_ok) {
    float* w = mrg + ((size_t)warp * a.G + hrow) * (D + 2);
    if (c4 == 0) {
      w[0] = m_run;
      w[1] = l;
    }
#pragma unroll
    for (int nn = 0; nn < NT; ++nn) {
      w[2 + 8 * nn + 2 * c4] = acc[nn][0] + acc[nn][2];
      w[3 + 8 * nn + 2 * c4] = acc[nn][1] + acc[nn][3];
    }
    if (warp == 0 && c4 == 0) x.used[(size_t)b * a.Hq + g * a.G + hrow] = used;
  }
  named_bar(1, NC * 32);
  for (int e = tid; e < a.G * D; e += NC * 32) {
    const int h = e / D, col = e % D;
    float M = -INFINITY;
    for (int w = 0; w < NC; ++w) M = fmaxf(M, mrg[((size_t)w * a.G + h) * (D + 2)]);
    float num = 0.f, den = 0.f;
    if (M != -INFINITY)
      for (int w = 0; w < NC; ++w) {
        const float* x = mrg + ((size_t)w * a.G + h) * (D + 2);
        const float f = exp2f(x[0] - M);
        den += x[1] * f;
        num += x[2 + col] * f;
      }
    a.out[((size_t)b * a.Hq + g * a.G + h) * D + col] = (den > 0.f) ? num / den : 0.f;
  }
}

}  // namespace nosa
