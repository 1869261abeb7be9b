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
constexpr int kSmallSel = 256;  // candidate sets up to this size use O(n^2) rank counting

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
  int* list;         // [kSmallSel] candidate indices (rank-count path)
  uint32_t* lkey;    // [kSmallSel] their keys
};

__host__ __device__ inline size_t sel_smem_bytes(int max_blocks) {
  const size_t nbp = (size_t)((max_blocks + 31) / 32) * 32;
  const size_t W = nbp / 32;
  return 4 * nbp + 6 * 4 * W + 4 * 256 + 4 * 33 + 4 * 8 + 8 * kSmallSel + 16;
}

// Offset of the score kernel's per-chunk values after the selection scratch (16-byte aligned).
__host__ __device__ inline size_t score_su_offset(int max_blocks) {
  return (sel_smem_bytes(max_blocks) + 15) & ~size_t(15);
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
  s.list = s.sc + 8;
  s.lkey = reinterpret_cast<uint32_t*>(s.list + kSmallSel);
  return s;
}

__device__ __forceinline__ uint32_t word_valid_mask(int w, int n) {
  const int lo = w * 32;
  if (n >= lo + 32) return 0xffffffffu;
  if (n <= lo) return 0u;
  return (1u << (n - lo)) - 1u;
}

// Exact top-m by radix select: the threshold key, 8 bits per pass with warp-aggregated
// histogram updates, then the lowest-index keys equal to the threshold fill the remainder.
// ORs the chosen bits into out[0..W) (out must be zeroed by the caller). Used when a
// range bucket holds more than kSmallSel keys (e.g. many equal scores).
__device__ void sel_topm_radix(const SelSmem& S, const uint32_t* cand, uint32_t* out, int W, int m) {
  const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31;
  uint32_t prefix = 0, pmask = 0;
  int rem = m;
  const int span = W * 32;
  const int iters = (span + nth - 1) / nth;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += nth) S.hist[i] = 0;
    __syncthreads();
    for (int it = 0; it < iters; ++it) {
      const int j = it * nth + tid;
      bool take = false;
      uint32_t dig = 0;
      if (j < span && ((cand[j >> 5] >> (j & 31)) & 1u)) {
        const uint32_t k = S.key[j];
        take = (k & pmask) == prefix;
        dig = (k >> shift) & 255u;
      }
      const unsigned act = __ballot_sync(0xffffffffu, take);
      if (take) {
        const unsigned peers = __match_any_sync(act, dig);
        if (lane == __ffs(peers) - 1) atomicAdd(&S.hist[dig], __popc(peers));
      }
    }
    __syncthreads();
    if (tid < 32) {
      int c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = S.hist[255 - 8 * tid - i];
        sum += c[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const int excl = incl - sum;
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
  const int eb = block_exclusive_scan(ne, S.red, nullptr);
  if (tid < W) {
    int take = rem - eb;
    take = take < 0 ? 0 : (take > ne ? ne : take);
    uint32_t t = eq, keep = 0;
    for (int x = 0; x < take; ++x) {
      const uint32_t low = t & (~t + 1u);
      keep |= low;
      t ^= low;
    }
    out[tid] |= gt | keep;
  }
  __syncthreads();
}

// Inverse of ord_f32 for keys of finite floats.
__device__ __forceinline__ float key_f32(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Bucket of a key among 256 over [kmin, kmax]. Any map that never decreases as the key grows
// keeps the selection exact: keys in a higher bucket are strictly larger than keys in a lower
// one, and the boundary bucket is ranked exactly. Float keys (scores) use equal-width buckets
// in value, so a bell-shaped set of scores spreads over many buckets and the boundary bucket
// holds a handful of keys; other keys use the top 8 bits of (key - kmin).
struct KeyBuckets {
  uint32_t kmin;
  int shift;
  float vlo, inv;
  bool lin;
  __device__ KeyBuckets(uint32_t lo, uint32_t hi, bool float_keys) : kmin(lo) {
    const uint32_t range = hi - lo;
    shift = (range < 256u) ? 0 : (32 - __clz(range) - 8);
    vlo = key_f32(lo);
    const float vhi = key_f32(hi), span = vhi - vlo;
    inv = 256.0f / span;
    lin = float_keys && isfinite(vlo) && isfinite(vhi) && span > 0.0f && isfinite(span) &&
          isfinite(inv) && inv > 0.0f;
  }
  __device__ __forceinline__ uint32_t operator()(uint32_t k) const {
    if (lin) return min(255u, static_cast<uint32_t>(__float2int_rz((key_f32(k) - vlo) * inv)));
    return (k - kmin) >> shift;
  }
};

// Top-m of key[] over the candidate bitmask cand[0..W): higher key first, equal keys to
// the lower index. Writes the bitmask into out[0..W). Returns min(m, |cand|).
// All threads of the CTA must call it; W <= blockDim.x. FLOAT_KEYS: the keys are ord_f32
// images of floats (scores); otherwise they may tie massively (LRU stamps), and the
// histogram, the boundary list and an all-equal boundary bucket are handled for that.
//  1. one pass: candidate count, smallest and largest key;
//  2. keys fall into 256 buckets spanning [min, max] (KeyBuckets), a histogram finds the
//     bucket holding the m-th key;
//  3. buckets above it are taken whole; the boundary bucket's keys are ranked exactly
//     against each other (or, if it holds more than kSmallSel keys, radix-selected).
template <bool FLOAT_KEYS>
__device__ int sel_topm(const SelSmem& S, const uint32_t* cand, uint32_t* out, int W, int m) {
  const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nw = nth >> 5;
  const int span = W * 32;
  // element-strided passes: the 32 lanes of a warp cover one bitmask word per iteration
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  int cnt = 0;
  for (int j = tid; j < span; j += nth) {
    if ((cand[j >> 5] >> (j & 31)) & 1u) {
      const uint32_t k = S.key[j];
      kmin = min(kmin, k);
      kmax = max(kmax, k);
      ++cnt;
    }
  }
  for (int i = tid; i < 256; i += nth) S.hist[i] = 0;
  // single-instruction warp reductions (redux.sync) instead of shuffle trees
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  cnt = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt)));
  uint32_t* ured = reinterpret_cast<uint32_t*>(S.red);
  if (lane == 0) {
    ured[warp] = kmin;
    ured[8 + warp] = kmax;
    S.red[16 + warp] = cnt;
  }
  if (tid == 0) S.sc[2] = 0;
  __syncthreads();
  int total = 0;
  kmin = 0xffffffffu;
  kmax = 0u;
  for (int i = 0; i < nw; ++i) {
    kmin = min(kmin, ured[i]);
    kmax = max(kmax, ured[8 + i]);
    total += S.red[16 + i];
  }
  if (m <= 0 || m >= total) {
    for (int w = tid; w < W; w += nth) out[w] = (m <= 0) ? 0u : cand[w];
    __syncthreads();
    return m <= 0 ? 0 : total;
  }
  const KeyBuckets bucket(kmin, kmax, FLOAT_KEYS);
  // histogram. Scores spread over the buckets and plain atomics rarely collide; other keys
  // (e.g. blocks last used at the same step) can pile into one bucket, so there a warp
  // whose keys share one bucket adds them with a single atomic.
  if constexpr (FLOAT_KEYS) {
    for (int j = tid; j < span; j += nth)
      if ((cand[j >> 5] >> (j & 31)) & 1u) atomicAdd(&S.hist[bucket(S.key[j])], 1);
  } else for (int j = tid; j < span; j += nth) {  // span is a multiple of 32: warp-uniform
    const bool in = (cand[j >> 5] >> (j & 31)) & 1u;
    const uint32_t bk = in ? bucket(S.key[j]) : 0u;
    const unsigned act = __ballot_sync(0xffffffffu, in);
    if (act) {
      const int lead = __ffs(act) - 1;
      const uint32_t b0 = __shfl_sync(0xffffffffu, bk, lead);
      if (__all_sync(0xffffffffu, !in || bk == b0)) {
        if (lane == lead) atomicAdd(&S.hist[b0], __popc(act));
      } else if (in) {
        atomicAdd(&S.hist[bk], 1);
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    int c[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = S.hist[255 - 8 * tid - i];
      sum += c[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += y;
    }
    const int excl = incl - sum;
    if (excl < m && m <= incl) {
      int acc = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (acc + c[i] >= m) {
          S.sc[0] = 255 - 8 * tid - i;  // boundary bucket
          S.sc[1] = m - acc;            // keys still to take from it
          S.sc[3] = c[i];               // its size
          break;
        }
        acc += c[i];
      }
    }
  }
  __syncthreads();
  const uint32_t bstar = static_cast<uint32_t>(S.sc[0]);
  const int rem = S.sc[1], nb = S.sc[3];
  const bool small = nb <= kSmallSel;
  for (int base = 0; base < span; base += nth) {
    const int j = base + tid;
    bool take = false, bnd = false;
    uint32_t k = 0u;
    if (j < span && ((cand[j >> 5] >> (j & 31)) & 1u)) {
      k = S.key[j];
      const uint32_t bk = bucket(k);
      take = bk > bstar;
      bnd = bk == bstar;
      if (FLOAT_KEYS && bnd && small) {
        const int slot = atomicAdd(&S.sc[2], 1);
        S.list[slot] = j;
        S.lkey[slot] = k;
      }
    }
    const uint32_t tw = __ballot_sync(0xffffffffu, take);
    const uint32_t bw = __ballot_sync(0xffffffffu, bnd);
    if (!FLOAT_KEYS && small && bw) {
      // tied keys: one atomic per warp reserves the warp's slots in the boundary list
      const int lead = __ffs(bw) - 1;
      int slot0 = 0;
      if (lane == lead) slot0 = atomicAdd(&S.sc[2], __popc(bw));
      slot0 = __shfl_sync(0xffffffffu, slot0, lead);
      if (bnd) {
        const int slot = slot0 + __popc(bw & ((1u << lane) - 1u));
        S.list[slot] = j;
        S.lkey[slot] = k;
      }
    }
    if (lane == 0 && j < span) {
      out[j >> 5] = tw;
      if (!small) S.m2[j >> 5] = bw;
    }
  }
  __syncthreads();
  if (small) {
    for (int t = tid; t < nb; t += nth) {
      const uint32_t k = S.lkey[t];
      const int j = S.list[t];
      int rank = 0;
#pragma unroll 8
      for (int u = 0; u < nb; ++u) {
        const uint32_t o = S.lkey[u];
        rank += (o > k) || (o == k && S.list[u] < j);
      }
      if (rank < rem) atomicOr(&out[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
  } else if constexpr (FLOAT_KEYS) {
    sel_topm_radix(S, S.m2, out, W, rem);
  } else {
    // The boundary bucket is too large to rank key against key. When all its keys are equal
    // (blocks last used at the same step) the lowest indices win, and a prefix count over
    // the bucket's mask words decides; otherwise radix select.
    uint32_t bmin = 0xffffffffu, bmax = 0u;
    for (int j = tid; j < span; j += nth) {
      if ((S.m2[j >> 5] >> (j & 31)) & 1u) {
        const uint32_t k = S.key[j];
        bmin = min(bmin, k);
        bmax = max(bmax, k);
      }
    }
    bmin = __reduce_min_sync(0xffffffffu, bmin);
    bmax = __reduce_max_sync(0xffffffffu, bmax);
    if (lane == 0) {
      ured[warp] = bmin;
      ured[8 + warp] = bmax;
    }
    __syncthreads();
    bmin = 0xffffffffu;
    bmax = 0u;
    for (int i = 0; i < nw; ++i) {
      bmin = min(bmin, ured[i]);
      bmax = max(bmax, ured[8 + i]);
    }
    __syncthreads();  // ured is reused by the scan below
    if (bmin == bmax) {
      const uint32_t bw = (tid < W) ? S.m2[tid] : 0u;
      const int before = block_exclusive_scan(__popc(bw), S.red, nullptr);
      if (tid < W) {
        int take = rem - before;
        take = take < 0 ? 0 : (take > __popc(bw) ? __popc(bw) : take);
        uint32_t t = bw, keep = 0u;
        for (int x = 0; x < take; ++x) {
          const uint32_t low = t & (~t + 1u);
          keep |= low;
          t ^= low;
        }
        out[tid] |= keep;
      }
      __syncthreads();
    } else {
      sel_topm_radix(S, S.m2, out, W, rem);
    }
  }
  return m;
}

// dst[0..W) = the bits of src[0..W) whose blocks are resident in HBM (block table entry >= 0);
// without host pools (bt NULL) every block is. Table entries are read one per thread, all of
// a pass in flight together, and each warp assembles one word with a ballot.
// All threads must call it; blockDim.x a multiple of 32.
__device__ void resident_bits(const uint32_t* src, uint32_t* dst, const int32_t* bt, int W) {
  const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, warp = tid >> 5;
  for (int j0 = 0; j0 < W * 32; j0 += nth) {
    const int j = j0 + tid;
    const bool in = j < W * 32 && ((src[j >> 5] >> (j & 31)) & 1u);
    const bool keep = in && (!bt || __ldcg(bt + j) >= 0);
    const uint32_t bw = __ballot_sync(0xffffffffu, keep);
    const int w = (j0 >> 5) + warp;
    if (lane == 0 && w < W) dst[w] = bw;
  }
  __syncthreads();
}

// Writes the set bits of mask[0..W) in ascending order to dst[rank]; returns |mask|.
// All threads must call it.
__device__ int sel_compact(const SelSmem& S, const uint32_t* mask, int W, int32_t* dst) {
  const int tid = threadIdx.x;
  if (W <= 32) {
    // one warp, no block-wide scan
    if (tid < 32) {
      const uint32_t mw = (tid < W) ? mask[tid] : 0u;
      const int c = __popc(mw);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      uint32_t t = mw;
      int r = incl - c;
      while (t) {
        const int b = __ffs(t) - 1;
        t &= t - 1;
        dst[r++] = tid * 32 + b;
      }
      if (tid == 31) S.sc[4] = incl;
    }
    __syncthreads();
    return S.sc[4];
  }
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

// Query-agnostic half of the dual selection for one group: Gamma_e = top-k_e of the
// eviction scores over C_e = S(t-1) & A(t-1); candidates left out leave A for good.
// Writes Gamma_e to ge_out (global, [Wmax] words) and updates alive. Returns |Gamma_e|.
__device__ int select_evict(const SelSmem& S, const float* evict, const uint32_t* prev, uint32_t* alive,
                            uint32_t* ge_out, int N, int k_e, int Wmax) {
  const int tid = threadIdx.x, nth = blockDim.x;
  const int W = (N + 31) / 32;
#pragma unroll 4
  for (int j = tid; j < N; j += nth) S.key[j] = ord_f32(__ldg(evict + j));
  for (int w = tid; w < Wmax; w += nth) {
    const uint32_t a = alive[w];
    S.m1[w] = a;
    S.cand[w] = prev[w] & a & word_valid_mask(w, N);
  }
  __syncthreads();
  const int ne = sel_topm<true>(S, S.cand, S.ge, W, k_e);
  for (int w = tid; w < Wmax; w += nth) {
    const uint32_t c = (w < W) ? S.cand[w] : 0u;
    const uint32_t g = (w < W) ? S.ge[w] : 0u;
    alive[w] = S.m1[w] & ~(c & ~g);
    if (ge_out) ge_out[w] = g;
  }
  __syncthreads();
  return ne;
}

// Query-aware half: Gamma_q = top-min(k - |Gamma_e|, N - |Gamma_e|) of the block scores over
// [0, N) minus Gamma_e, S(t) = Gamma_e + Gamma_q written to prev and, ascending and padded
// with -1, to sel. Gamma_e comes from ge (global words written earlier in the same launch by
// another CTA) or, when ge is NULL, from S.ge. On return S.sset holds S(t).
__device__ void select_query(const SelSmem& S, const float* scores, const uint32_t* ge, uint32_t* prev,
                             int32_t* sel, int N, int k, int Wmax) {
  const int tid = threadIdx.x, nth = blockDim.x;
  const int W = (N + 31) / 32;
  int ne = 0;
  for (int w = tid; w < W; w += nth) {
    const uint32_t g = ge ? __ldcg(ge + w) : S.ge[w];
    S.ge[w] = g;
    S.cand[w] = word_valid_mask(w, N) & ~g;
    ne += __popc(g);
  }
#pragma unroll 4
  for (int j = tid; j < N; j += nth) S.key[j] = ord_f32(__ldcg(scores + j));
  for (int o = 16; o >= 1; o >>= 1) ne += __shfl_xor_sync(0xffffffffu, ne, o);
  if ((tid & 31) == 0) S.red[tid >> 5] = ne;
  __syncthreads();
  ne = 0;
  for (int i = 0; i < (nth >> 5); ++i) ne += S.red[i];
  __syncthreads();
  const int mq = (k - ne < N - ne) ? k - ne : N - ne;
  sel_topm<true>(S, S.cand, S.pick, W, mq);
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
  // need (m1), resident (m2), misses (cand). Global tables are read element-strided, one
  // entry per thread, and each warp assembles one 32-bit word per pass with a ballot: all
  // loads of a pass are in flight together instead of one dependent load per block.
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int U = 8;  // loads in flight per thread
  for (int j00 = 0; j00 < W * 32; j00 += U * nth) {
    int pg[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j00 + u * nth + tid;
      pg[u] = (j < N) ? p.block_table[j] : -1;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j0 = j00 + u * nth;
      if (j0 >= W * 32) break;
      bool res = false;
      if (pg[u] >= 0) {
        if (pg[u] < p.page_base || pg[u] >= p.page_base + p.slots) set_err(p.err, NOSA_ERR_BLOCK_TABLE);
        else res = true;
      }
      const uint32_t rw = __ballot_sync(0xffffffffu, res);
      const int w = (j0 >> 5) + warp;
      if (lane == 0 && w < W) {
        uint32_t need = S.sset[w];
        if ((tail >> 5) == w) need |= 1u << (tail & 31);
        S.m1[w] = need;
        S.m2[w] = rw;
        S.cand[w] = need & ~rw;
      }
    }
  }
  __syncthreads();
  int nmiss = 0;
  if (tid < W) nmiss = __popc(S.cand[tid]);
  const int nm = block_sum(nmiss, S.red);
  // free slots -> pick (bitmask over slots)
  int nfr = 0;
  for (int z00 = 0; z00 < Wf * 32; z00 += U * nth) {
    int ow[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int z = z00 + u * nth + tid;
      ow[u] = (z < p.slots) ? p.slot_owner[z] : 0;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int z0 = z00 + u * nth;
      if (z0 >= Wf * 32) break;
      const bool f = ow[u] < 0;
      const uint32_t fw = __ballot_sync(0xffffffffu, f);
      const int w = (z0 >> 5) + warp;
      if (lane == 0 && w < Wf) S.pick[w] = fw;
      nfr += f ? 1 : 0;
    }
  }
  const int nfree = block_sum(nfr, S.red);
  const int nf_use = nm < nfree ? nm : nfree;
  int nv = nm - nf_use;
  // victims -> ge (reused as the victim bitmask)
  if (nv > 0) {
    if (tid < W) S.m2[tid] = S.m2[tid] & ~S.m1[tid];  // evictable
    __syncthreads();
    for (int j00 = 0; j00 < W * 32; j00 += U * nth) {
      int lu[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j00 + u * nth + tid;
        lu[u] = (j < W * 32 && ((S.m2[j >> 5] >> (j & 31)) & 1u)) ? p.last_used[j] : 0;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j00 + u * nth + tid;
        if (j < W * 32 && ((S.m2[j >> 5] >> (j & 31)) & 1u)) S.key[j] = ord_lru(lu[u]);
      }
    }
    __syncthreads();
    const int got = sel_topm<false>(S, S.m2, S.ge, W, nv);
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
    }
    for (int j = tid; j < W * 32; j += nth)
      if ((S.m1[j >> 5] >> (j & 31)) & 1u) p.last_used[j] = p.L;
    if (tid == 0) {
      *p.copy_count = nassign;
      if (p.miss_count) *p.miss_count = nm;
    }
    __syncthreads();
  }
}

}  // namespace nosa
