// The offline teacher cache: per row of teacher logits, the K most likely
// tokens and their log-probabilities.
//
// "Дистилляция LLM на одной GPU: offline-кэш и chunked KL loss", section
// «Два приёма»: the teacher runs once, the 100 most likely tokens of every
// position are kept, and training reads that cache.  This is the step that
// writes it, given the teacher's logits.
//
// One CTA per row (persistent over rows).  The streaming form (below, K up
// to its TS_THREADS = 256 threads) reads each row once from HBM and once more
// from L2.  The histogram form, used for larger K and for rows the streaming form
// cannot settle, makes three passes over the row (the first from HBM, the
// others mostly from L2):
//   1. the largest logit (packed bf16 maxima, two per instruction);
//   2. the row's sum of exp(z - max) (log-sum-exp = max + log of it), and a
//      histogram of the 128 keys just below the largest (one bucket per bf16
//      value, one binade) whose block scan finds the K-th largest key; only
//      if fewer than K elements fall there does the window slide down, 4096
//      keys at a time, in further passes;
//   3. every element at or above that key is gathered, and a bitonic sort of
//      (key, -id) in shared memory puts them in order: descending logit,
//      equal logits by smaller id.
// Keys are the bf16 bit patterns mapped to an order-preserving 16-bit code
// (-0 counts as +0), so every comparison is exact.  The passes compare the
// values themselves (bf16 widens exactly; key order is value order) and form
// a key only for the elements that enter the histogram or the candidates,
// which keeps the instruction count per logit low: the kernel reads each
// logit once from HBM and is otherwise bound by its issue rate.
#pragma once

#include <cstdint>

#include "ckl_ptx.cuh"

#define CKL_DEV_TOPK_TIES 8  // more elements tie at the K-th logit than the sort holds

namespace ckl {

constexpr int TK_THREADS = 512;
constexpr int TK_WIN = 4096;  // keys per histogram window
constexpr int TK_WIN0 = 128;  // keys in the first window (one binade of bf16)
constexpr int TK_CAP = 2048;  // elements the final sort holds (K plus the ties at the K-th)

__device__ __forceinline__ uint32_t bf16_key(uint32_t b) {
  if (b == 0x8000u) b = 0u;  // -0 == +0
  return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  const uint32_t b = (k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu);
  return __uint_as_float(b << 16);
}

// Order-preserving keys of two packed bf16 values (each half as bf16_key).
__device__ __forceinline__ uint32_t bf16_key2(uint32_t w) {
  w &= ~__vcmpeq2(w, 0x80008000u);                 // -0 -> +0
  const uint32_t neg = ((w & 0x80008000u) >> 15) * 0x7FFFu;
  return w ^ (0x80008000u | neg);
}

constexpr int TK_UNROLL = 2;  // independent 16-byte loads in flight per thread
#ifndef CKL_TS_UNROLL
#define CKL_TS_UNROLL 4
#endif
constexpr int TS_UNROLL = CKL_TS_UNROLL;  // the same, in the streaming form's pass

__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Largest logit of the row (packed bf16 maxima, two per instruction).
__device__ __forceinline__ float tk_row_max(const uint16_t* z, int V, bool vec8) {
  float m = -INFINITY;
  if (vec8) {
    const uint4* z4 = reinterpret_cast<const uint4*>(z);
    const int n8 = V / 8;
    uint32_t m2 = 0xFF80FF80u;  // -inf, -inf
    for (int base = threadIdx.x; base < n8; base += TK_THREADS * TK_UNROLL) {
      uint4 v[TK_UNROLL];
#pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int i = base + u * TK_THREADS;
        v[u] = (i < n8) ? z4[i] : make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
      }
#pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u)
        m2 = bf16x2_max(m2, bf16x2_max(bf16x2_max(v[u].x, v[u].y), bf16x2_max(v[u].z, v[u].w)));
    }
    m = fmaxf(bf16_lo(m2), bf16_hi(m2));
  } else {
    for (int i = threadIdx.x; i < V; i += TK_THREADS)
      m = fmaxf(m, __uint_as_float(static_cast<uint32_t>(z[i]) << 16));
  }
  return m;
}

// Calls f(value, raw bf16 bits, id) for every element of the row, eight bf16
// per 16-byte load when the row allows it.  The id is a constant offset from
// the load's index, so it costs nothing where f does not use it.
template <typename F>
__device__ __forceinline__ void tk_for_row(const uint16_t* z, int V, bool vec8, F&& f) {
  if (vec8) {
    const uint4* z4 = reinterpret_cast<const uint4*>(z);
    const int n8 = V / 8;
    for (int base = threadIdx.x; base < n8; base += TK_THREADS * TK_UNROLL) {
      uint4 v[TK_UNROLL];
#pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int i = base + u * TK_THREADS;
        if (i < n8) v[u] = z4[i];
      }
#pragma unroll
      for (int u = 0; u < TK_UNROLL; ++u) {
        const int i = base + u * TK_THREADS;
        if (i < n8) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            f(bf16_lo(w[j]), w[j] & 0xFFFFu, 8 * i + 2 * j);
            f(bf16_hi(w[j]), w[j] >> 16, 8 * i + 2 * j + 1);
          }
        }
      }
    }
  } else {
    for (int i = threadIdx.x; i < V; i += TK_THREADS) {
      const uint32_t b = z[i];
      f(__uint_as_float(b << 16), b, i);
    }
  }
}

// Shared memory of one row's selection (histogram form).
struct TkShared {
  uint32_t hist[TK_WIN];
  unsigned long long cand[TK_CAP];
  float s_s[TK_THREADS / 32];
  float s_c[TK_THREADS / 32];
  uint32_t s_part[TK_THREADS / 32];
  uint32_t s_thr, s_ncand, s_found, s_total;
  float s_lse;
};

// Sorts the row's n candidates (key << 32 | ~id) in shared memory, descending
// (equal keys: smaller id first), and writes the first K: ids and z - lse.
// NT = threads of the block.
template <int NT = TK_THREADS, typename SM>
__device__ __forceinline__ void tk_sort_and_write(SM& sm, uint32_t n, int K, float lse,
                                                  int64_t row, int32_t* idx_out,
                                                  float* logp_out) {
  const int tid = threadIdx.x;
  uint32_t P = 1;
  while (P < n) P <<= 1;
  for (uint32_t i = n + tid; i < P; i += NT) sm.cand[i] = 0ull;
  __syncthreads();
  for (uint32_t k = 2; k <= P; k <<= 1) {
    for (uint32_t j = k >> 1; j > 0; j >>= 1) {
      for (uint32_t i = tid; i < P; i += NT) {
        const uint32_t ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = sm.cand[i], b = sm.cand[ixj];
          const bool up = (i & k) == 0;
          if (up ? (a < b) : (a > b)) { sm.cand[i] = b; sm.cand[ixj] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int k = tid; k < K; k += NT) {
    const unsigned long long e = sm.cand[k];
    const uint32_t key = static_cast<uint32_t>(e >> 32);
    idx_out[row * K + k] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(e));
    logp_out[row * K + k] = key_value(key) - lse;
  }
  __syncthreads();
}

// Adds element i (value v, bf16 bits raw) to the candidates if v >= v_thr.
template <typename SM>
__device__ __forceinline__ void tk_put(SM& sm, float v, uint32_t raw, int i, float v_thr) {
  if (v >= v_thr) {
    const uint32_t slot = atomicAdd(&sm.s_ncand, 1u);
    if (slot < TK_CAP)
      sm.cand[slot] = (static_cast<unsigned long long>(bf16_key(raw)) << 32) |
                      (0xFFFFFFFFu - static_cast<uint32_t>(i));
  }
}

// Gathers every element of the row whose value is >= v_thr into the
// candidates; returns their count (the array holds at most TK_CAP).
template <int NT = TK_THREADS, int UNROLL = TK_UNROLL, typename SM>
__device__ __forceinline__ uint32_t tk_gather(SM& sm, const uint16_t* z, int V, bool vec8,
                                              float v_thr) {
  if (threadIdx.x == 0) sm.s_ncand = 0;
  __syncthreads();
  auto put = [&](float v, uint32_t raw, int i) { tk_put(sm, v, raw, i, v_thr); };
  if (vec8) {
    // a whole 8-element vector below the threshold is skipped on its maximum
    const uint4* z4 = reinterpret_cast<const uint4*>(z);
    const int n8 = V / 8;
    for (int base = threadIdx.x; base < n8; base += NT * UNROLL) {
      uint4 v[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int i = base + u * NT;
        if (i < n8) v[u] = z4[i];
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int i = base + u * NT;
        if (i >= n8) continue;
        const uint32_t m2 = bf16x2_max(bf16x2_max(v[u].x, v[u].y), bf16x2_max(v[u].z, v[u].w));
        if (fmaxf(bf16_lo(m2), bf16_hi(m2)) < v_thr) continue;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          put(bf16_lo(w[j]), w[j] & 0xFFFFu, 8 * i + 2 * j);
          put(bf16_hi(w[j]), w[j] >> 16, 8 * i + 2 * j + 1);
        }
      }
    }
  } else {
    for (int i = threadIdx.x; i < V; i += NT) {
      const uint32_t b = z[i];
      put(__uint_as_float(b << 16), b, i);
    }
  }
  __syncthreads();
  return sm.s_ncand;
}

// One row by histogram windows (exact for any data with at most TK_CAP
// elements at or above the K-th largest value): the largest logit; the sum of
// exp against it and the histogram of the 128 keys just below it, sliding
// down 4096 keys at a time until K elements are covered; the gather; the sort.
__device__ void tk_row_hist(TkShared& sm, const uint16_t* z, int V, bool vec8, int K,
                            int64_t row, int32_t* idx_out, float* logp_out, int* status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- pass 1: the largest logit
  float zm = tk_row_max(z, V, vec8);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) zm = fmaxf(zm, __shfl_xor_sync(0xffffffffu, zm, o));
  if (lane == 0) sm.s_s[warp] = zm;
  for (int j = tid; j < TK_WIN; j += TK_THREADS) sm.hist[j] = 0;
  if (tid == 0) { sm.s_found = 0; sm.s_thr = 0; }
  __syncthreads();
  float zmax = -INFINITY;
  for (int w = 0; w < TK_THREADS / 32; ++w) zmax = fmaxf(zmax, sm.s_s[w]);
  __syncthreads();  // s_s is reused below
  // its key (bf16 bits of the value; -0 counts as +0)
  const uint32_t kmax = bf16_key(__float_as_uint(zmax) >> 16);

  // ---- pass 2: sum of exp against the maximum, and the first window's
  // histogram; further windows (4096 keys each) only when needed
  uint32_t above = 0;         // elements with a key above the window
  int top = static_cast<int>(kmax);
  float lse = 0.f;
  for (int win = 0;; ++win) {
    const int lo = top - (win == 0 ? TK_WIN0 : TK_WIN) + 1;
    // the window's bounds as values: key order is value order
    const float v_lo = lo > 0 ? key_value(static_cast<uint32_t>(lo)) : -INFINITY;
    const float v_top = key_value(static_cast<uint32_t>(top));
    if (win == 0) {
      float s = 0.f;
      tk_for_row(z, V, vec8, [&](float v, uint32_t raw, int) {
        s += ex2_approx((v - zmax) * LOG2E);  // v - zmax is exact near the max
        if (v >= v_lo) atomicAdd(&sm.hist[top - static_cast<int>(bf16_key(raw))], 1u);
      });
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) sm.s_s[warp] = s;
    } else {
      for (int j = tid; j < TK_WIN; j += TK_THREADS) sm.hist[j] = 0;
      __syncthreads();
      tk_for_row(z, V, vec8, [&](float v, uint32_t raw, int) {
        if (v <= v_top && v >= v_lo) atomicAdd(&sm.hist[top - static_cast<int>(bf16_key(raw))], 1u);
      });
    }
    __syncthreads();
    if (win == 0) {
      float S = 0.f;
      for (int w = 0; w < TK_THREADS / 32; ++w) S += sm.s_s[w];
      lse = zmax + logf(S);
    }
    // block scan over the window: thread tid owns buckets [8 tid, 8 tid + 8)
    uint32_t own = 0;
#pragma unroll
    for (int j = 0; j < TK_WIN / TK_THREADS; ++j) own += sm.hist[tid * (TK_WIN / TK_THREADS) + j];
    uint32_t incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) sm.s_part[warp] = incl;
    __syncthreads();
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += sm.s_part[w];
    before += incl - own;  // elements in buckets before this thread's (higher keys)
    if (tid == TK_THREADS - 1) sm.s_total = before + own;
    if (above + before < static_cast<uint32_t>(K) &&
        above + before + own >= static_cast<uint32_t>(K)) {
      uint32_t c = above + before;
      for (int j = 0; j < TK_WIN / TK_THREADS; ++j) {
        c += sm.hist[tid * (TK_WIN / TK_THREADS) + j];
        if (c >= static_cast<uint32_t>(K)) {
          sm.s_thr = static_cast<uint32_t>(top - (tid * (TK_WIN / TK_THREADS) + j));
          sm.s_found = 1;
          break;
        }
      }
    }
    __syncthreads();
    if (sm.s_found || lo <= 0) break;
    above += sm.s_total;
    top = lo - 1;
    __syncthreads();
  }
  const float v_thr = key_value(sm.s_thr);

  // ---- pass 3: gather every element at or above the threshold, sort
  const uint32_t ncand = tk_gather(sm, z, V, vec8, v_thr);
  if (tid == 0 && ncand > static_cast<uint32_t>(TK_CAP) && status != nullptr)
    atomicOr(status, CKL_DEV_TOPK_TIES);
  tk_sort_and_write(sm, min(ncand, static_cast<uint32_t>(TK_CAP)), K, lse, row, idx_out,
                    logp_out);
}

__global__ void __launch_bounds__(TK_THREADS, 2)
topk_cache_kernel(const uint16_t* __restrict__ logits, int64_t T, int V, int K, int vec8,
                  int32_t* __restrict__ idx_out, float* __restrict__ logp_out, int* status) {
  __shared__ TkShared sm;
  for (int64_t row = blockIdx.x; row < T; row += gridDim.x)
    tk_row_hist(sm, logits + row * static_cast<int64_t>(V), V, vec8 != 0, K, row, idx_out,
                logp_out, status);
}

// ------------------------------------------------------------ streaming form
// One read of the row from HBM.  Pass 1: every thread keeps its running
// maximum c and the sum of 2^((z - c) log2 e) over its own elements,
// rescaled when c grows (at most once per 8-element vector), and writes each
// of its vectors' maximum (a bf16) to shared memory; the block merges the
// (c, sum) pairs into the row's log-sum-exp.  The K-th largest of the
// threads' maxima is at most the row's K-th largest value (those K maxima
// are K elements of the row), so it is a valid threshold.  Pass 2 scans the
// vector maxima in shared memory, lists the vectors whose maximum reaches the
// threshold (about 130 of the row's 16 032 at V = 128 256) and loads them
// again, one per thread; their elements at or above it are the candidates,
// and each candidate's rank among them (their keys are distinct) places the
// first K in order.  With the row's top K spread over the threads, the
// threshold sits just below the K-th value and a few more than K elements are
// gathered.  When more than TS_MARKS vectors are marked or more than TK_CAP
// elements would be gathered (the row's large values crowded into few
// threads, or heavy ties), the row is marked and done again by histogram
// windows in topk_fallback_kernel.  Rows whose vector maxima do not fit the dynamic
// shared memory the launch gives (V above TS_MARK_MAX_V), or whose length is
// not a multiple of 8, gather by reading the row again instead.  Blocks of
// TS_THREADS threads, up to TS_BLOCKS per SM; needs K <= TS_THREADS.
#ifndef CKL_TS_THREADS
#define CKL_TS_THREADS 256
#endif
constexpr int TS_THREADS = CKL_TS_THREADS;
#ifndef CKL_TS_BLOCKS
#define CKL_TS_BLOCKS 4
#endif
constexpr int TS_BLOCKS = CKL_TS_BLOCKS;  // blocks per SM (at most)
constexpr int TS_MARK_MAX_V = 262144;     // vector maxima of up to 64 KB per block

constexpr int TS_MARKS = 512;  // marked vectors a row may have (more: the fallback)

struct alignas(16) TsShared {
  unsigned long long cand[TK_CAP];
  uint32_t keys[TS_THREADS];  // the threads' maximum keys, for the threshold
  uint32_t marked[TS_MARKS];  // indices of the vectors pass 2 loads again
  uint32_t s_nmarked;
  float s_c[TS_THREADS / 32];
  float s_s[TS_THREADS / 32];
  float s_lse;
  uint32_t s_thr, s_ncand;
};

// The K-th largest of the block's keys (one per thread; 0 = no element),
// or 0 when fewer than K are non-zero.  The keys go to shared memory and
// warp 0 selects the answer bit by bit from the most significant: at each
// bit it counts, with ballots, the keys that agree with the bits chosen so
// far and have this one set; if at least the remaining rank are, the answer
// has the bit, otherwise those keys all rank above it.  Called by one warp
// on the keys in sm.keys.
__device__ __forceinline__ uint32_t ts_kth_key_warp(const TsShared& sm, int K) {
  constexpr int KPL = TS_THREADS / 32;  // keys per lane
  const int lane = threadIdx.x & 31;
  uint32_t k[KPL];
#pragma unroll
  for (int j = 0; j < KPL; ++j) k[j] = sm.keys[j * 32 + lane];
  uint32_t mine = 0;
#pragma unroll
  for (int j = 0; j < KPL; ++j) mine += (k[j] != 0u) ? 1u : 0u;
  uint32_t prefix = 0;
  if (__reduce_add_sync(0xffffffffu, mine) >= static_cast<uint32_t>(K)) {
    uint32_t need = static_cast<uint32_t>(K);
#pragma unroll 1
    for (int bit = 15; bit >= 0; --bit) {
      const uint32_t hi = (prefix >> bit) | 1u;  // the chosen bits, then this one set
      uint32_t c = 0;
#pragma unroll
      for (int j = 0; j < KPL; ++j) c += ((k[j] >> bit) == hi) ? 1u : 0u;
      const uint32_t cnt = __reduce_add_sync(0xffffffffu, c);
      if (cnt >= need) prefix |= 1u << bit;
      else need -= cnt;
    }
  }
  return prefix;
}


// The vector maxima of a row, as pass 1 leaves them: for each of a thread's
// passes over TS_UNROLL x TS_THREADS vectors, its TS_UNROLL = 4 maxima (bf16
// bits, -inf past the row's end) packed into one uint2 at [pass][thread], so
// that a thread writes and reads its own four with one 8-byte access.
static_assert(TS_UNROLL == 4, "the packed vector maxima hold four per thread and pass");
constexpr int TS_PER_PASS = TS_THREADS * TS_UNROLL;  // vectors per pass of the block

// Pass 2 from the vector maxima.  Each thread scans its own packed maxima
// (four compared at once, one bf16x2 max) and lists the vectors whose maximum
// reaches v_thr; then the block loads the listed vectors, one per thread, so
// that the loads of a row are in flight together, and gathers their elements
// at or above v_thr.  Returns the number of candidates, or TK_CAP + 1 when
// more than TS_MARKS vectors are marked (the row then goes to the fallback).
template <typename SM>
__device__ __forceinline__ uint32_t ts_gather_marked(SM& sm, const uint2* vmax,
                                                     const uint16_t* z, int n8, float v_thr) {
  if (threadIdx.x == 0) { sm.s_ncand = 0; sm.s_nmarked = 0; }
  __syncthreads();
  const int passes = (n8 + TS_PER_PASS - 1) / TS_PER_PASS;
  for (int it = 0; it < passes; ++it) {
    const uint2 e = vmax[it * TS_THREADS + threadIdx.x];
    const uint32_t m = bf16x2_max(e.x, e.y);
    if (fmaxf(bf16_lo(m), bf16_hi(m)) < v_thr) continue;
#pragma unroll
    for (int u = 0; u < TS_UNROLL; ++u) {
      const uint32_t word = (u < 2) ? e.x : e.y;
      const float vm = (u & 1) ? bf16_hi(word) : bf16_lo(word);
      const int i = it * TS_PER_PASS + u * TS_THREADS + threadIdx.x;
      if (vm >= v_thr && i < n8) {
        const uint32_t slot = atomicAdd(&sm.s_nmarked, 1u);
        if (slot < static_cast<uint32_t>(TS_MARKS)) sm.marked[slot] = static_cast<uint32_t>(i);
      }
    }
  }
  __syncthreads();
  const uint32_t nm = sm.s_nmarked;
  if (nm > static_cast<uint32_t>(TS_MARKS)) return TK_CAP + 1;  // uniform over the block
  const uint4* z4 = reinterpret_cast<const uint4*>(z);
  for (uint32_t k = threadIdx.x; k < nm; k += TS_THREADS) {
    const int i = static_cast<int>(sm.marked[k]);
    const uint4 v = z4[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      tk_put(sm, bf16_lo(w[j]), w[j] & 0xFFFFu, 8 * i + 2 * j, v_thr);
      tk_put(sm, bf16_hi(w[j]), w[j] >> 16, 8 * i + 2 * j + 1, v_thr);
    }
  }
  __syncthreads();
  return sm.s_ncand;
}

// Packed pairs of fp32 (lane 0 in the low word), for the sm_100 two-lane
// add / sub / mul instructions.
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float f32x2_lo(uint64_t r) { return __uint_as_float(static_cast<uint32_t>(r)); }
__device__ __forceinline__ float f32x2_hi(uint64_t r) { return __uint_as_float(static_cast<uint32_t>(r >> 32)); }
__device__ __forceinline__ uint64_t bf16x2_widen(uint32_t w) {  // both halves, exactly
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Per-thread pass-1 state of one row: running maximum and sum of exp.
struct TsAcc {
  float cmax = -INFINITY;  // this thread's largest value so far
  float s = 0.f;           // sum of 2^((z - cmax) log2 e)
  __device__ __forceinline__ void rescale(float vm) {
    if (vm > cmax) {
      s *= ex2_approx((cmax - vm) * LOG2E);  // 0 while nothing was summed
      cmax = vm;
    }
  }
  // one 8-element vector; returns its maximum
  __device__ __forceinline__ float add8(const uint4& v) {
    const uint32_t m2 = bf16x2_max(bf16x2_max(v.x, v.y), bf16x2_max(v.z, v.w));
    const float vm = fmaxf(bf16_lo(m2), bf16_hi(m2));
    rescale(vm);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    // (z - cmax) log2 e for the two halves of a word at once (packed fp32
    // pairs, each lane rounded as the scalar form); z - cmax is exact for
    // the values that matter (near the maximum)
    const uint64_t c2 = f32x2_pack(cmax, cmax), l2 = f32x2_pack(LOG2E, LOG2E);
    uint64_t ab = 0;  // (+0, +0): the sums of the low and the high halves
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint64_t d = f32x2_mul(f32x2_sub(bf16x2_widen(w[j]), c2), l2);
      ab = f32x2_add(ab, f32x2_pack(ex2_approx(f32x2_lo(d)), ex2_approx(f32x2_hi(d))));
    }
    s += f32x2_lo(ab) + f32x2_hi(ab);
    return vm;
  }
};

// Writes the first K of the row's n candidates in order (descending value,
// equal values by smaller id: the candidates' keys are distinct) by ranking:
// each candidate counts the candidates above it, and the one of rank r < K
// writes output r.  One barrier instead of a sort's log^2; n <= 2 TS_THREADS.
template <typename SM>
__device__ __forceinline__ void ts_rank_and_write(SM& sm, uint32_t n, int K, float lse,
                                                  int64_t row, int32_t* idx_out,
                                                  float* logp_out) {
  const ulonglong2* c2 = reinterpret_cast<const ulonglong2*>(sm.cand);
  for (uint32_t c = threadIdx.x; c < n; c += TS_THREADS) {
    const unsigned long long mine = sm.cand[c];
    uint32_t rank = (n & 1u) && sm.cand[n - 1] > mine ? 1u : 0u;
#pragma unroll 4
    for (uint32_t q = 0; q < n / 2; ++q) {  // two candidates per 16-byte read
      const ulonglong2 e = c2[q];
      rank += (e.x > mine ? 1u : 0u) + (e.y > mine ? 1u : 0u);
    }
    if (rank < static_cast<uint32_t>(K)) {
      idx_out[row * K + rank] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(mine));
      logp_out[row * K + rank] = key_value(static_cast<uint32_t>(mine >> 32)) - lse;
    }
  }
  __syncthreads();
}

// The end of a row once every thread has its pass-1 state: log-sum-exp,
// threshold, gather (from the vector maxima when vmax is given), sort, write.
__device__ __forceinline__ void ts_finish_row(TsShared& sm, const TsAcc& acc, const uint16_t* z,
                                              int V, bool vec8, const uint2* vmax, int K,
                                              int64_t row, int32_t* idx_out, float* logp_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float wc = acc.cmax, ws = acc.s;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float oc = __shfl_xor_sync(0xffffffffu, wc, o);
    const float os = __shfl_xor_sync(0xffffffffu, ws, o);
    const float nc = fmaxf(wc, oc);
    ws = (nc == -INFINITY) ? 0.f
                           : ws * ex2_approx((wc - nc) * LOG2E) + os * ex2_approx((oc - nc) * LOG2E);
    wc = nc;
  }
  if (lane == 0) { sm.s_c[warp] = wc; sm.s_s[warp] = ws; }
  // the threshold, the K-th largest of the threads' maxima, by warp 0 while
  // warp 1 merges the warps' (max, sum) pairs into the row's log-sum-exp
  sm.keys[threadIdx.x] = (acc.cmax == -INFINITY) ? 0u : bf16_key(__float_as_uint(acc.cmax) >> 16);
  __syncthreads();
  if (warp == 0) {
    const uint32_t t = ts_kth_key_warp(sm, K);
    if (lane == 0) sm.s_thr = t;
  } else if (warp == 1 && lane == 0) {
    float C = -INFINITY;
    for (int w = 0; w < TS_THREADS / 32; ++w) C = fmaxf(C, sm.s_c[w]);
    float S = 0.f;
    for (int w = 0; w < TS_THREADS / 32; ++w) S += sm.s_s[w] * ex2_approx((sm.s_c[w] - C) * LOG2E);
    sm.s_lse = C + logf(S);
  }
  __syncthreads();
  const uint32_t thr = sm.s_thr;
  const float lse = sm.s_lse;
  const float v_thr = (thr == 0u) ? -INFINITY : key_value(thr);
  const uint32_t ncand = vmax ? ts_gather_marked(sm, vmax, z, V / 8, v_thr)
                              : tk_gather<TS_THREADS, TS_UNROLL>(sm, z, V, vec8, v_thr);
  if (ncand <= static_cast<uint32_t>(TK_CAP)) {
    if (ncand >= static_cast<uint32_t>(K) && ncand <= 2u * TS_THREADS)
      ts_rank_and_write(sm, ncand, K, lse, row, idx_out, logp_out);
    else
      tk_sort_and_write<TS_THREADS>(sm, ncand, K, lse, row, idx_out, logp_out);
  } else if (threadIdx.x == 0) {
    idx_out[row * K] = -1;  // left to topk_fallback_kernel
  }
}

// Pass 1 of rows of 8-element vectors: TS_UNROLL independent 16-byte loads in
// flight per thread, then their arithmetic.
__global__ void __launch_bounds__(TS_THREADS, TS_BLOCKS)
topk_stream_kernel(const uint16_t* __restrict__ logits, int64_t T, int V, int K, int vec8,
                   int mark, int32_t* __restrict__ idx_out, float* __restrict__ logp_out,
                   int* status) {
  __shared__ TsShared sm;
  // the packed vector maxima of the row when mark != 0 (then vec8 != 0)
  extern __shared__ uint2 ts_vmax[];
  const int tid = threadIdx.x;
  for (int64_t row = blockIdx.x; row < T; row += gridDim.x) {
    const uint16_t* z = logits + row * static_cast<int64_t>(V);
    TsAcc acc;
    if (vec8) {
      const uint4* z4 = reinterpret_cast<const uint4*>(z);
      const int n8 = V / 8;
      int it = 0;
      for (int base = tid; base < n8; base += TS_PER_PASS, ++it) {
        uint4 v[TS_UNROLL];
#pragma unroll
        for (int u = 0; u < TS_UNROLL; ++u) {
          const int i = base + u * TS_THREADS;
          if (i < n8) v[u] = z4[i];
        }
        uint32_t mb[TS_UNROLL];
#pragma unroll
        for (int u = 0; u < TS_UNROLL; ++u) {
          mb[u] = 0xFF80u;  // -inf: past the row's end
          if (base + u * TS_THREADS < n8) mb[u] = __float_as_uint(acc.add8(v[u])) >> 16;
        }
        if (mark) ts_vmax[it * TS_THREADS + tid] = make_uint2(mb[0] | (mb[1] << 16), mb[2] | (mb[3] << 16));
      }
      // a thread whose first vector is past the row's end still owns the
      // entries of the passes it skipped
      if (mark)
        for (int k = it; k * TS_PER_PASS < n8; ++k)
          ts_vmax[k * TS_THREADS + tid] = make_uint2(0xFF80FF80u, 0xFF80FF80u);
    } else {
      for (int i = tid; i < V; i += TS_THREADS) {
        const float v = __uint_as_float(static_cast<uint32_t>(z[i]) << 16);
        acc.rescale(v);
        acc.s += ex2_approx((v - acc.cmax) * LOG2E);
      }
    }
    ts_finish_row(sm, acc, z, V, vec8 != 0, mark ? ts_vmax : nullptr, K, row, idx_out, logp_out);
  }
}

// The rows topk_stream_kernel left (first id -1), by histogram windows.  A
// kernel of its own, so that the streaming kernel's registers are not shaped
// by a path it rarely takes.
__global__ void __launch_bounds__(TK_THREADS, 2)
topk_fallback_kernel(const uint16_t* __restrict__ logits, int64_t T, int V, int K, int vec8,
                     int32_t* __restrict__ idx_out, float* __restrict__ logp_out, int* status) {
  __shared__ TkShared sm;
  // the block's rows are checked in parallel (one load each), TK_THREADS at a time
  for (int64_t first = blockIdx.x; first < T; first += static_cast<int64_t>(gridDim.x) * TK_THREADS) {
    const int64_t mine = first + static_cast<int64_t>(threadIdx.x) * gridDim.x;
    const bool left = mine < T && idx_out[mine * K] == -1;
    if (!__syncthreads_or(left)) continue;
    __shared__ uint32_t s_left[TK_THREADS / 32];
    const uint32_t bits = __ballot_sync(0xffffffffu, left);
    if ((threadIdx.x & 31) == 0) s_left[threadIdx.x >> 5] = bits;
    __syncthreads();
    for (int t = 0; t < TK_THREADS; ++t) {
      if (!((s_left[t >> 5] >> (t & 31)) & 1u)) continue;  // uniform over the block
      const int64_t row = first + static_cast<int64_t>(t) * gridDim.x;
      tk_row_hist(sm, logits + row * static_cast<int64_t>(V), V, vec8 != 0, K, row, idx_out,
                  logp_out, status);
    }
    __syncthreads();
  }
}

}  // namespace ckl
