// Per-group dual selection and residency planning, run by one CTA (256 threads)
// of the score kernel's last-arriving chunk, or by the standalone kernels.
//
// NOSA (gist.science/es/paper/2510.13602), "Metodologia" 1: query-aware set
// Gamma_q, query-agnostic eviction set Gamma_e with the never-again rule,
// locality bound gamma(t) >= k_e/k; "Metodologia" 2: set differences decide the
// blocks to swap. Sets are bitmasks over the group's blocks; top-m is an exact
// radix select on 32-bit order-preserving keys with ties to the lower index.
#pragma once

#include "nosa_common.cuh"

namespace nosa {

constexpr int kSelThreads = 256;

// Shared-memory scratch of the selection, carved from dynamic shared memory.
struct SelSmem {
  uint32_t* key;     // [round_up(max_blocks, 32)]; reused as the slot list in planning
  uint32_t* cand;    // [W] candidate bitmask
  uint32_t* pick;    // [W] chosen by the last top-m
  uint32_t* ge;      // [W] Gamma_e
  uint32_t* sset;    // [W] S(t)
  uint32_t* m1;      // [W] scratch mask
  uint32_t* m2;      // [W] scratch mask
  int* hist;         // [256]
  int* red;          // [33]
  int* sc;           // [8]
};

__host__ __device__ inline size_t sel_smem_bytes(int max_blocks) {
  const size_t nbp = (size_t)((max_blocks + 31) / 32) * 32;
  const size_t W = nbp / 32;
  return 4 * nbp + 6 * 4 * W + 4 * 256 + 4 * 33 + 4 * 8 + 16;
}

__device__ inline SelSmem sel_smem_carve(uint8_t* base, int max_blocks) {
  const int nbp = ((max_blocks + 31) / 32) * 32;
  const int W = nbp / 32;
  SelSmem s;
  uint32_t* p = reinterpret_cast<uint32_t*>(base);
  s.key = p; p += nbp;
  s.cand = p; p += W;
  s.pick = p; p += W;
  s.ge = p; p += W;
  s.sset = p; p += W;
  s.m1 = p; p += W;
  s.m2 = p; p += W;
  s.hist = reinterpret_cast<int*>(p);
  s.red = s.hist + 256;
  s.sc = s.red + 33;
  return s;
}

__device__ __forceinline__ uint32_t word_valid_mask(int w, int n) {
  const int lo = w * 32;
  if (n >= lo + 32) return 0xffffffffu;
  if (n <= lo) return 0u;
  return (1u << (n - lo)) - 1u;
}

// Top-m of key[] over the candidate bitmask cand[0..W): higher key first, equal keys to
// the lower index. Writes the bitmask into out[0..W). Returns min(m, |cand|).
// All threads of the CTA must call it; W <= blockDim.x.
__device__ int sel_topm(const SelSmem& S, const uint32_t* cand, uint32_t* out, int W, int m) {
  const int tid = threadIdx.x, nth = blockDim.x;
  int cnt = 0;
  for (int w = tid; w < W; w += nth) cnt += __popc(cand[w]);
  const int total = block_sum(cnt, S.red);
  if (m <= 0 || m >= total) {
    for (int w = tid; w < W; w += nth) out[w] = (m <= 0) ? 0u : cand[w];
    __syncthreads();
    return m <= 0 ? 0 : total;
  }
  uint32_t prefix = 0, pmask = 0;
  int rem = m;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += nth) S.hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < W * 32; j += nth) {
      if ((cand[j >> 5] >> (j & 31)) & 1u) {
        const uint32_t k = S.key[j];
        if ((k & pmask) == prefix) atomicAdd(&S.hist[(k >> shift) & 255u], 1);
      }
    }
    __syncthreads();
    if (tid < 32) {
      // lane owns bins 255-8*lane .. 248-8*lane (descending key order)
      int c[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = S.hist[255 - 8 * tid - i];
        s += c[i];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const int excl = incl - s;
      if (excl < rem && rem <= incl) {
        int acc = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc + c[i] >= rem) {
            S.sc[0] = 255 - 8 * tid - i;
            S.sc[1] = rem - acc;
            break;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(S.sc[0]) << shift;
    pmask |= 0xffu << shift;
    rem = S.sc[1];
    __syncthreads();
  }
  // keys above the threshold, plus the `rem` lowest-index keys equal to it
  uint32_t gt = 0, eq = 0;
  if (tid < W) {
    const uint32_t cw = cand[tid];
    for (int b = 0; b < 32; ++b) {
      if ((cw >> b) & 1u) {
        const uint32_t k = S.key[tid * 32 + b];
        gt |= static_cast<uint32_t>(k > prefix) << b;
        eq |= static_cast<uint32_t>(k == prefix) << b;
      }
    }
  }
  const int ne = __popc(eq);
  const int before = block_exclusive_scan(ne, S.red, nullptr);
  if (tid < W) {
    int take = rem - before;
    take = take < 0 ? 0 : (take > ne ? ne : take);
    uint32_t t = eq, keep = 0;
    for (int x = 0; x < take; ++x) {
      const uint32_t low = t & (~t + 1u);
      keep |= low;
      t ^= low;
    }
    out[tid] = gt | keep;
  }
  __syncthreads();
  return m;
}

// Writes the set bits of mask[0..W) in ascending order to dst[base + rank]; returns |mask|.
__device__ int sel_compact(const SelSmem& S, const uint32_t* mask, int W, int32_t* dst) {
  const int tid = threadIdx.x;
  const uint32_t mw = (tid < W) ? mask[tid] : 0u;
  int total;
  const int before = block_exclusive_scan(__popc(mw), S.red, &total);
  if (tid < W) {
    uint32_t t = mw;
    int r = before;
    while (t) {
      const int b = __ffs(t) - 1;
      t &= t - 1;
      dst[r++] = tid * 32 + b;
    }
  }
  __syncthreads();
  return total;
}

// Dual selection of one group. scores/evict: the group's rows (global). prev/alive: the
// group's bitmask words (global, updated). sel: the group's k outputs. On return S.sset
// holds S(t).
__device__ void select_group(const SelSmem& S, const float* scores, const float* evict,
                             uint32_t* prev, uint32_t* alive, int32_t* sel, int N, int k_e, int k,
                             int Wmax) {
  const int tid = threadIdx.x, nth = blockDim.x;
  const int W = (N + 31) / 32;
  for (int w = tid; w < Wmax; w += nth) {
    const uint32_t a = alive[w];
    S.m1[w] = a;
    S.cand[w] = prev[w] & a & word_valid_mask(w, N);
  }
  for (int j = tid; j < N; j += nth) S.key[j] = ord_f32(__ldg(evict + j));
  __syncthreads();
  const int ne = sel_topm(S, S.cand, S.ge, W, k_e);
  // candidates left out of Gamma_e leave the alive set for good
  for (int w = tid; w < Wmax; w += nth) {
    const uint32_t c = (w < W) ? S.cand[w] : 0u;
    const uint32_t g = (w < W) ? S.ge[w] : 0u;
    alive[w] = S.m1[w] & ~(c & ~g);
    if (w < W) S.cand[w] = word_valid_mask(w, N) & ~g;
  }
  for (int j = tid; j < N; j += nth) S.key[j] = ord_f32(__ldcg(scores + j));
  __syncthreads();
  const int mq = (k - ne < N - ne) ? k - ne : N - ne;
  sel_topm(S, S.cand, S.pick, W, mq);
  for (int w = tid; w < Wmax; w += nth) {
    const uint32_t s = (w < W) ? (S.ge[w] | S.pick[w]) : 0u;
    S.sset[w] = s;
    prev[w] = s;
  }
  __syncthreads();
  const int n = sel_compact(S, S.sset, W, sel);
  for (int i = n + tid; i < k; i += nth) sel[i] = -1;
  __syncthreads();
}

// Loads S(t) from a sel list (ascending or not) into S.sset.
__device__ void sset_from_list(const SelSmem& S, const int32_t* sel, int k, int N, int Wmax,
                               uint32_t* err) {
  const int tid = threadIdx.x, nth = blockDim.x;
  for (int w = tid; w < Wmax; w += nth) S.sset[w] = 0u;
  __syncthreads();
  for (int i = tid; i < k; i += nth) {
    const int j = sel[i];
    if (j >= 0 && j < N) atomicOr(&S.sset[j >> 5], 1u << (j & 31));
    else if (j >= N) set_err(err, NOSA_ERR_SEL);
  }
  __syncthreads();
}

struct PlanArgs {
  int32_t* block_table;   // group row [max_blocks]
  int32_t* slot_owner;    // group row [slots]
  int32_t* last_used;     // group row [max_blocks]
  int2* copy_list;        // group row (block, page)
  int32_t* copy_count;    // &copy_count[gi]
  int32_t* miss_count;    // &miss_count[gi] or nullptr
  uint32_t* err;
  int L, bs, slots, page_base, max_blocks;
};

// Residency of one group given S(t) in S.sset: misses = (S + tail) minus resident; free
// slots first, then least-recently-used victims outside S + tail (ascending block order).
__device__ void plan_group(const SelSmem& S, const PlanArgs& p) {
  const int tid = threadIdx.x, nth = blockDim.x;
  const int N = (p.L + p.bs - 1) / p.bs;
  const int W = (N + 31) / 32;
  const int tail = (p.L - 1) / p.bs;
  const int Wf = (p.slots + 31) / 32;
  // need (m1), resident (m2)
  if (tid < W) {
    uint32_t need = S.sset[tid];
    if ((tail >> 5) == tid) need |= 1u << (tail & 31);
    uint32_t res = 0;
    for (int b = 0; b < 32; ++b) {
      const int j = tid * 32 + b;
      if (j >= N) break;
      const int pg = p.block_table[j];
      if (pg >= 0) {
        if (pg < p.page_base || pg >= p.page_base + p.slots) set_err(p.err, NOSA_ERR_BLOCK_TABLE);
        else res |= 1u << b;
      }
    }
    S.m1[tid] = need;
    S.m2[tid] = res;
    S.cand[tid] = need & ~res;  // misses
  }
  __syncthreads();
  int nmiss = 0;
  if (tid < W) nmiss = __popc(S.cand[tid]);
  const int nm = block_sum(nmiss, S.red);
  // free slots -> pick (bitmask over slots)
  int nfr = 0;
  for (int w = tid; w < Wf; w += nth) {
    uint32_t f = 0;
    for (int b = 0; b < 32; ++b) {
      const int z = w * 32 + b;
      if (z < p.slots && p.slot_owner[z] < 0) f |= 1u << b;
    }
    S.pick[w] = f;
    nfr += __popc(f);
  }
  const int nfree = block_sum(nfr, S.red);
  const int nf_use = nm < nfree ? nm : nfree;
  int nv = nm - nf_use;
  // victims -> ge (reused as the victim bitmask)
  if (nv > 0) {
    if (tid < W) S.m2[tid] = S.m2[tid] & ~S.m1[tid];  // evictable
    for (int w = tid; w < W; w += nth) {
      const uint32_t v = S.m2[w];
      for (int b = 0; b < 32; ++b)
        if ((v >> b) & 1u) S.key[w * 32 + b] = ord_lru(p.last_used[w * 32 + b]);
    }
    __syncthreads();
    const int got = sel_topm(S, S.m2, S.ge, W, nv);
    if (got < nv) {
      set_err(p.err, NOSA_ERR_NO_VICTIM);
      nv = got;
    }
  } else {
    for (int w = tid; w < W; w += nth) S.ge[w] = 0u;
    __syncthreads();
  }
  // slot list (S.key reused): free slots ascending, then the victims' slots
  {
    const uint32_t f = (tid < Wf) ? S.pick[tid] : 0u;
    const int before = block_exclusive_scan(__popc(f), S.red, nullptr);
    if (tid < Wf) {
      uint32_t t = f;
      int r = before;
      while (t && r < nf_use) {
        const int b = __ffs(t) - 1;
        t &= t - 1;
        S.key[r++] = static_cast<uint32_t>(tid * 32 + b);
      }
    }
    const uint32_t v = (tid < W) ? S.ge[tid] : 0u;
    const int vb = block_exclusive_scan(__popc(v), S.red, nullptr);
    if (tid < W) {
      uint32_t t = v;
      int r = nf_use + vb;
      while (t) {
        const int b = __ffs(t) - 1;
        t &= t - 1;
        const int j = tid * 32 + b;
        S.key[r++] = static_cast<uint32_t>(p.block_table[j] - p.page_base);
        p.block_table[j] = -1;
      }
    }
    __syncthreads();
  }
  // misses ascending take the slots in order
  {
    const uint32_t mw = (tid < W) ? S.cand[tid] : 0u;
    const int before = block_exclusive_scan(__popc(mw), S.red, nullptr);
    const int nassign = nf_use + nv;
    if (tid < W) {
      uint32_t t = mw;
      int r = before;
      while (t) {
        const int b = __ffs(t) - 1;
        t &= t - 1;
        if (r < nassign) {
          const int j = tid * 32 + b;
          const int z = static_cast<int>(S.key[r]);
          const int page = p.page_base + z;
          p.block_table[j] = page;
          p.slot_owner[z] = j;
          p.copy_list[r] = make_int2(j, page);
        }
        ++r;
      }
      const uint32_t need = S.m1[tid];
      for (int b = 0; b < 32; ++b)
        if ((need >> b) & 1u) p.last_used[tid * 32 + b] = p.L;
    }
    if (tid == 0) {
      *p.copy_count = nassign;
      if (p.miss_count) *p.miss_count = nm;
    }
    __syncthreads();
  }
}

}  // namespace nosa
