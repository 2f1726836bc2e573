// Device kernels of the fused chunked KL-distillation loss (sm_100a).
//
// The method (Multiverse Computing, "Efficient Knowledge Distillation for
// LLMs: Offline Top-K Logits and a Fused Chunked KL Loss", as summarised in
// "LLMのための効率的な知識蒸留：オフラインTop-K LogitsおよびFused Chunked KL
// Loss", section "2つのシステム変更"): project one chunk of hidden states to
// logits, fold the chunk into the running loss, drop it; the backward
// recomputes each chunk.  Here:
//
//   prep      per row: check the cached ids, renormalise the K teacher
//             log-probs (p = softmax over K), sum p log p, sort (id, p) by id,
//             count the positions that count (N).
//   tc<FWD>   Z = H W^T on tcgen05 (TMEM accumulators, TMA-fed), never
//             stored: the epilogue keeps a running max / sum of exp per row
//             and gathers z at the row's teacher ids (sum_k p_k z_{idx_k}),
//             one partial per (row, vocabulary split).
//   combine   merges the splits: lse_t, KL_t = sum p log p - sum p z + lse,
//             the masked mean (fixed-order sums, deterministic).
//   tc<DZ>    per chunk: recomputes the same Z tiles (same instruction
//             sequence, so bit-identical z), dZ = exp(z - lse) - scatter(p)
//             for rows that count (0 otherwise), stored bf16 as 64-column
//             panels [V/64][chunk][64] so every later read of it is contiguous.
//   tc<DHDW>  per chunk, one persistent launch: dH_c = s dZ_c W (A K-major,
//             B MN-major) and dW (+)= s dZ_c^T H_c (A = dZ^T MN-major, B =
//             H_c^T K-major from a transposed copy), s = g/N, written by TMA
//             store / TMA reduce-add.
#pragma once

#include <cfloat>
#include <climits>
#include <cstdint>

#include "ckl_ptx.cuh"

// DHDW: alternate the k direction of a slot's consecutive jobs (1) or not (0).
#ifndef CKL_SERPENTINE
#define CKL_SERPENTINE 1
#endif

namespace ckl {

constexpr int BM = 128;           // rows per tile (TMEM lanes)
constexpr int BK = 64;            // bf16 elements per 128-byte swizzle row (32 for fp32)
constexpr int BN_V = 256;         // vocabulary columns per logit tile
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES = 256 * BK * 2;       // 32 KB (largest B tile)
constexpr int EPI_STAGE = BM * 128;         // one 128-row x 128-byte staging tile, 16 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = 256;          // TMEM columns per accumulator buffer

// FWD: logits + online log-sum-exp + teacher gather; DZ: logit recompute +
// dZ; DHDW: dH and dW of one chunk; FWDZ: FWD over one chunk that also
// stores the fp32 logits (the single-pass schedule).
enum Mode { MODE_FWD = 0, MODE_DZ = 1, MODE_DHDW = 2, MODE_FWDZ = 3 };

// Pipeline depth and epilogue width.  A single CTA holds a 128 x 256 tile:
// four 48 KB operand stages fill the shared memory beside the epilogue
// staging.  A CTA pair (PAIR) shares one 256-row MMA: each CTA stages its own
// 128 rows of A and half of B, 32 KB per stage, so six stages fit.  Four
// epilogue warps, one per TMEM lane group (eight, splitting the columns,
// measured slower: the extra staging costs an operand stage, and the
// epilogue is not the bottleneck).
template <int MODE, bool PAIR>
struct Cfg {
  static constexpr int STAGES = PAIR ? 6 : 4;
  static constexpr int EPI_WARPS = 4;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int B_STAGE = PAIR ? B_BYTES / 2 : B_BYTES;
  static constexpr int MB = PAIR ? 2 * BM : BM;  // rows of one job's M extent
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = STAGES * A_BYTES;
  static constexpr int EPI_OFF = B_OFF + STAGES * B_STAGE;
  static constexpr int BAR_OFF = EPI_OFF + 2 * EPI_STAGE;  // two staging tiles
  static constexpr int SMEM_ALLOC = BAR_OFF + 256 + 1024;  // + slack to align the base to 1 KB
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(8 * (2 * STAGES + 9) + 4 <= 256, "barrier area");
};

constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct alignas(64) TcParams {
  CUtensorMap tm[6];
  int32_t T, d, V, K;
  int32_t rows;     // FWD: T; DZ / DHDW: rows of this chunk
  int32_t row0;     // DZ / DHDW: first row of this chunk
  int32_t n_rb;     // row blocks of 128 (FWD: over T; DZ / DHDW: over the chunk)
  int32_t n_vt;     // vocabulary tiles of 256
  int32_t S;        // vocabulary splits (FWD / DZ)
  int32_t n_units;  // FWD: n_rb * S units; DZ: n_rb * n_vt tiles
  int32_t bn;       // DHDW: d-tile width (64, 128, 192 or 256)
  int32_t n_nt;     // DHDW: d tiles
  int32_t n_mt;     // DHDW: vocabulary tiles of 128 (dW rows)
  int32_t n5, n6;   // DHDW: dH units, dW units
  int32_t c5, c6;   // DHDW: k-blocks per dH unit (over V), per dW unit (over rows)
  int32_t dw_store; // DHDW: 1 = this block stores dW, 0 = adds into it
  int32_t vt0;      // FWD / DZ: first vocabulary tile of this launch's slab
  int32_t v_lo;     // DHDW: first vocabulary column of this launch's slab
  int32_t dh_mode;  // DHDW: 0 = dH as bf16, 1 = store fp32 partial dH, 2 = add into it
  int32_t dw_mode;  // DHDW: 0 = contiguous dW ranges per slot, 1 = dW tiles dealt in rounds
  int32_t split_fast;  // FWD: units numbered split-fastest (see JobIter)
  int32_t dw_Ql, dw_El, dw_Qh, dw_Eh;  // DHDW rounds: quotas, see JobIter
  int32_t v_off;    // FWD / DZ: teacher id of local vocabulary column 0 (a vocabulary shard)
  int32_t w3d;      // DHDW: tm[1] is the 3-D view of W (one box per stage for the dH B operand)
  const int2* pairs;      // [T, K] (id, p as bits), sorted by id per row
  float4* partials;       // FWD: [T, S] (max of z log2e, sum 2^(..), sum p z, 0)
  const float* lse;       // DZ: [T]
  const uint8_t* mask;    // [T] or null (every position counts)
  const float* grad_loss; // DHDW: [1] or null (= 1)
  int* status;            // device status word
  const int* countN;      // N = number of positions that count
};

// ------------------------------------------------------------------ prep
// One warp per row; K <= 256 (at most 8 entries per lane).
constexpr int PREP_WARPS = 8;
constexpr int PREP_MAXK = 256;

__global__ void __launch_bounds__(PREP_WARPS * 32)
prep_kernel(const int32_t* __restrict__ idx, const float* __restrict__ logp,
            const uint8_t* __restrict__ mask, int64_t T, int K, int64_t V,
            int2* __restrict__ pairs, float* __restrict__ Hp, int* status, int* countN) {
  __shared__ int s_id[PREP_WARPS][PREP_MAXK];
  __shared__ int s_cnt[PREP_WARPS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * PREP_WARPS + warp;
  int counts = 0;
  int flags = 0;
  if (t < T) {
    int id[8];
    float lp[8];
    const int64_t base = t * K;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = lane + 32 * e;
      id[e] = INT_MAX;
      lp[e] = -INFINITY;
      if (k < K) {
        int v = idx[base + k];
        float l = logp[base + k];
        if (v < 0 || static_cast<int64_t>(v) >= V) {
          flags |= CKL_DEV_BAD_INDEX;
          v = INT_MAX;  // never matches a vocabulary column
          l = -INFINITY;
        }
        if (isnan(l) || l == INFINITY) {
          flags |= CKL_DEV_BAD_LOGP;
          l = -INFINITY;
        }
        id[e] = v;
        lp[e] = l;
      }
    }
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, lp[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (m == -INFINITY) {
      flags |= CKL_DEV_BAD_LOGP;  // no finite log-prob in this row
      m = 0.f;
    }
    float se = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) se += (lp[e] == -INFINITY) ? 0.f : expf(lp[e] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
    const float ell = m + logf(se);
    float p[8];
    float hp = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      p[e] = (lp[e] == -INFINITY) ? 0.f : expf(lp[e] - ell);
      hp += (p[e] > 0.f) ? p[e] * (lp[e] - ell) : 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) hp += __shfl_xor_sync(0xffffffffu, hp, o);
    // Sort by (id, original position): rank = number of entries before it.
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = lane + 32 * e;
      if (k < K) s_id[warp][k] = id[e];
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = lane + 32 * e;
      if (k < K) {
        int rank = 0;
        for (int j = 0; j < K; ++j) {
          const int o = s_id[warp][j];
          rank += (o < id[e]) || (o == id[e] && j < k);
        }
        pairs[base + rank] = make_int2(id[e], __float_as_int(p[e]));
      }
    }
    if (lane == 0) {
      Hp[t] = hp;
      counts = (mask == nullptr || mask[t] != 0) ? 1 : 0;
    }
  }
  if (lane == 0) s_cnt[warp] = counts;
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0 && flags) atomicOr(status, flags);
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int w = 0; w < PREP_WARPS; ++w) c += s_cnt[w];
    if (c) atomicAdd(countN, c);
  }
}

// The same for 256 < K <= PREP_MAXK_LARGE: one 256-thread CTA per row; the
// (id, position) keys are put in order by a bitonic sort in shared memory,
// which gives the warp kernel's order (id, then position in the cache).
constexpr int PREPL_THREADS = 256;
constexpr int PREP_MAXK_LARGE = 2048;

__device__ __forceinline__ float prepl_block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = -INFINITY;
  for (int w = 0; w < PREPL_THREADS / 32; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}
__device__ __forceinline__ float prepl_block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < PREPL_THREADS / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

// The smallest row of idx [T, K] that holds some id more than once, by
// atomicMin into *first_dup_row (pre-set to -1, i.e. 0xFFFFFFFF unsigned).
// One CTA per row, persistent; the row's ids in shared memory, each thread
// comparing its ids with every later one (K^2 / 2 comparisons per row).
constexpr int DUP_THREADS = 256;
__global__ void __launch_bounds__(DUP_THREADS)
dup_ids_kernel(const int32_t* __restrict__ idx, int64_t T, int K, uint32_t* first_dup_row) {
  __shared__ int32_t ids[PREP_MAXK_LARGE];
  __shared__ int s_found;
  for (int64_t row = blockIdx.x; row < T; row += gridDim.x) {
    if (threadIdx.x == 0) s_found = 0;
    for (int k = threadIdx.x; k < K; k += DUP_THREADS) ids[k] = idx[row * K + k];
    __syncthreads();
    bool dup = false;
    for (int a = threadIdx.x; a < K && !dup; a += DUP_THREADS) {
      const int32_t v = ids[a];
      for (int b = a + 1; b < K; ++b)
        if (ids[b] == v) { dup = true; break; }
    }
    if (dup) s_found = 1;
    __syncthreads();
    if (threadIdx.x == 0 && s_found) atomicMin(first_dup_row, static_cast<uint32_t>(row));
    __syncthreads();
  }
}


__global__ void __launch_bounds__(PREPL_THREADS)
prep_large_kernel(const int32_t* __restrict__ idx, const float* __restrict__ logp,
                  const uint8_t* __restrict__ mask, int64_t T, int K, int64_t V,
                  int2* __restrict__ pairs, float* __restrict__ Hp, int* status, int* countN) {
  __shared__ unsigned long long key[PREP_MAXK_LARGE];  // id << 32 | position
  __shared__ float lps[PREP_MAXK_LARGE];
  __shared__ float red[PREPL_THREADS / 32];
  const int tid = threadIdx.x;
  const int64_t t = blockIdx.x;
  const int64_t base = t * K;
  int flags = 0;
  for (int k = tid; k < K; k += PREPL_THREADS) {
    int v = idx[base + k];
    float l = logp[base + k];
    if (v < 0 || static_cast<int64_t>(v) >= V) {
      flags |= CKL_DEV_BAD_INDEX;
      v = INT_MAX;  // never matches a vocabulary column
      l = -INFINITY;
    }
    if (isnan(l) || l == INFINITY) {
      flags |= CKL_DEV_BAD_LOGP;
      l = -INFINITY;
    }
    key[k] = (static_cast<unsigned long long>(static_cast<uint32_t>(v)) << 32) |
             static_cast<uint32_t>(k);
    lps[k] = l;
  }
  int P = 1;
  while (P < K) P <<= 1;
  for (int k = K + tid; k < P; k += PREPL_THREADS) key[k] = ~0ull;
  __syncthreads();
  // renormalisation over the K entries
  float m = -INFINITY;
  for (int k = tid; k < K; k += PREPL_THREADS) m = fmaxf(m, lps[k]);
  m = prepl_block_max(m, red);
  if (m == -INFINITY) {
    flags |= CKL_DEV_BAD_LOGP;  // no finite log-prob in this row
    m = 0.f;
  }
  float se = 0.f;
  for (int k = tid; k < K; k += PREPL_THREADS) se += (lps[k] == -INFINITY) ? 0.f : expf(lps[k] - m);
  const float ell = m + logf(prepl_block_sum(se, red));
  float hp = 0.f;
  for (int k = tid; k < K; k += PREPL_THREADS) {
    const float pk = (lps[k] == -INFINITY) ? 0.f : expf(lps[k] - ell);
    hp += (pk > 0.f) ? pk * (lps[k] - ell) : 0.f;
  }
  hp = prepl_block_sum(hp, red);
  // bitonic sort of the keys, ascending: id, then position
  for (int k2 = 2; k2 <= P; k2 <<= 1) {
    for (int j = k2 >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += PREPL_THREADS) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = key[i], b = key[ixj];
          const bool up = (i & k2) == 0;
          if (up ? (a > b) : (a < b)) { key[i] = b; key[ixj] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int k = tid; k < K; k += PREPL_THREADS) {
    const unsigned long long e = key[k];
    const int pos = static_cast<int>(e & 0xFFFFFFFFull);
    const float l = lps[pos];
    const float pk = (l == -INFINITY) ? 0.f : expf(l - ell);
    pairs[base + k] = make_int2(static_cast<int>(e >> 32), __float_as_int(pk));
  }
  if (tid == 0) {
    Hp[t] = hp;
    if (mask == nullptr || mask[t] != 0) atomicAdd(countN, 1);
  }
  flags = __reduce_or_sync(0xffffffffu, flags);
  if ((tid & 31) == 0 && flags) atomicOr(status, flags);
}

// ------------------------------------------------------------------ combine
constexpr int COMBINE_THREADS = 256;

// Partial s of row t is partials[t * row_stride + s * split_stride]: the
// forward's vocabulary splits ([T][S]: S, 1) or the vocabulary shards of
// several GPUs gathered as [g][T] (1, T).
__global__ void __launch_bounds__(COMBINE_THREADS)
combine_kernel(const float4* __restrict__ partials, int S, int64_t row_stride,
               int64_t split_stride, const float* __restrict__ Hp,
               const uint8_t* __restrict__ mask, int64_t T, float* __restrict__ lse,
               double* block_sums, unsigned int* ticket, const int* countN, float* loss,
               double* numer) {
  __shared__ double s_w[COMBINE_THREADS / 32];
  __shared__ bool s_last;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * COMBINE_THREADS + threadIdx.x;
  float contrib = 0.f;
  if (t < T) {
    const float4* pr = partials + t * row_stride;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, pr[s * split_stride].x);
    float se = 0.f, pz = 0.f;
    for (int s = 0; s < S; ++s) {
      const float4 q = pr[s * split_stride];
      se += q.y * exp2f(q.x - M);
      pz += q.z;
    }
    const float l = (M + log2f(se)) * LN2;
    lse[t] = l;
    if (mask == nullptr || mask[t] != 0) contrib = Hp[t] - pz + l;
  }
  double v = static_cast<double>(contrib);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double b = 0.0;
    for (int w = 0; w < COMBINE_THREADS / 32; ++w) b += s_w[w];
    block_sums[blockIdx.x] = b;
    __threadfence();
    s_last = (atomicAdd(ticket, 1u) == gridDim.x - 1);
  }
  __syncthreads();
  if (s_last && threadIdx.x == 0) {
    __threadfence();
    double total = 0.0;
    const volatile double* bs = block_sums;
    for (unsigned b = 0; b < gridDim.x; ++b) total += bs[b];
    const int n = *reinterpret_cast<const volatile int*>(countN);
    *loss = (n > 0) ? static_cast<float>(total / static_cast<double>(n)) : 0.f;
    *numer = total;
  }
}

// One vocabulary shard's row partials: the forward's S splits of row t merged
// into (max of z log2e, sum of 2^(z log2e - max), sum of p z over the shard's
// teacher ids, 0), for the combine across shards.
__global__ void __launch_bounds__(COMBINE_THREADS)
merge_splits_kernel(const float4* __restrict__ partials, int S, int64_t T,
                    float4* __restrict__ out) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * COMBINE_THREADS + threadIdx.x;
  if (t >= T) return;
  const float4* pr = partials + t * S;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, pr[s].x);
  float se = 0.f, pz = 0.f;
  for (int s = 0; s < S; ++s) {
    const float4 q = pr[s];
    se += q.y * exp2f(q.x - M);
    pz += q.z;
  }
  out[t] = make_float4(M, se, pz, 0.f);
}

// H_c^T for the dW GEMM: Hc [rows, d] (pitch d) -> HcT [d, pitch_t] (rows
// contiguous), 32 x 32 tiles through shared memory.  E = uint16_t (bf16) or
// float (the fp32 entry points).
template <typename E>
__global__ void __launch_bounds__(256)
transpose_rows_kernel(const E* __restrict__ Hc, int rows, int d, E* __restrict__ HcT,
                      int pitch_t) {
  __shared__ E tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int r = r0 + ty + i, c = c0 + tx;
    if (r < rows && c < d) tile[ty + i][tx] = Hc[static_cast<int64_t>(r) * d + c];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int c = c0 + ty + i, r = r0 + tx;
    if (r < rows && c < d) HcT[static_cast<int64_t>(c) * pitch_t + r] = tile[tx][ty + i];
  }
}

// Loss of an empty batch (T = 0).
__global__ void zero_loss_kernel(float* loss) { *loss = 0.f; }

// Data parallel, after the forward on this rank's rows: (sum of KL over the
// rank's positions that count, N_r), twice: one copy for the sum over
// ranks, one kept.
__global__ void dp_local_stats_kernel(const double* numer, const int* countN, double* stats) {
  const double n = static_cast<double>(*countN);
  stats[0] = *numer;
  stats[1] = n;
  stats[2] = *numer;
  stats[3] = n;
}

// Data parallel, after stats[0..1] were summed over the ranks: the global
// mean loss, and the upstream gradient this rank's backward takes so that
// its own 1 / N_r scale becomes g / N (0 when no position counts anywhere).
__global__ void dp_finish_kernel(const double* stats, const float* grad_loss, float* loss,
                                 float* grad_local) {
  const double num = stats[0], n = stats[1], n_r = stats[3];
  const double g = (grad_loss != nullptr) ? static_cast<double>(*grad_loss) : 1.0;
  *loss = (n > 0.0) ? static_cast<float>(num / n) : 0.f;
  *grad_local = (n > 0.0) ? static_cast<float>(g * n_r / n) : 0.f;
}

// Self-test of the bounded waits: one CTA waits, with the kernels' own wait,
// on an mbarrier that nothing arrives on.  The wait runs out after limit_ns,
// records CKL_DEV_TIMEOUT in *status and the kernel returns normally, so the
// context stays usable.
__global__ void wait_timeout_selftest_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_ns(b, 0, status, limit_ns);
  __syncthreads();
}

// ------------------------------------------------------------------ single pass
// One chunk row per CTA, after the FWDZ GEMM: merge the row's vocabulary
// splits into lse_t and its loss term m_t (Hp_t - pz_t + lse_t), then turn the
// stored fp32 logits into dZ_t = m_t (exp(z - lse_t) - scatter p_t) as bf16 in
// the 64-column panel layout the dH/dW GEMM reads (columns V .. round_up(V, 64)
// are written 0): panel rows of pitch `cap`, this chunk's rows from `drow0`
// (several chunks share one dH/dW launch).  Same arithmetic as the recompute
// path's dZ epilogue.
constexpr int ZROW_THREADS = 512;
constexpr int ZROW_UNROLL = 4;

__global__ void __launch_bounds__(ZROW_THREADS)
zrow_kernel(const float* __restrict__ Z, int64_t zpitch, const float4* __restrict__ partials,
            int S, const float* __restrict__ Hp, const uint8_t* __restrict__ mask,
            const int2* __restrict__ pairs, int K, int V, int64_t row0, int64_t cap,
            int64_t drow0, float* __restrict__ lse, float* __restrict__ rowloss,
            uint16_t* __restrict__ dz) {
  __shared__ float s_lse2;
  __shared__ int s_counts;
  const int r = blockIdx.x;
  const int64_t t = row0 + r;
  const int64_t dr = drow0 + r;  // row within the dZ panels
  if (threadIdx.x == 0) {
    const float4* pr = partials + t * S;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, pr[s].x);
    float se = 0.f, pz = 0.f;
    for (int s = 0; s < S; ++s) {
      const float4 q = pr[s];
      se += q.y * exp2f(q.x - M);
      pz += q.z;
    }
    const float l = (M + log2f(se)) * LN2;
    const int counts = (mask == nullptr || mask[t] != 0) ? 1 : 0;
    lse[t] = l;
    rowloss[t] = counts ? Hp[t] - pz + l : 0.f;
    s_lse2 = l * LOG2E;
    s_counts = counts;
  }
  __syncthreads();
  const float lse2 = s_lse2;
  const bool counts = s_counts != 0;
  const float* zr = Z + static_cast<int64_t>(r) * zpitch;
  const int vend = (V + 63) & ~63;
  // softmax part, four columns per thread and load; ZROW_UNROLL loads in
  // flight per thread before any of them is used
  for (int v0 = 4 * threadIdx.x; v0 < vend; v0 += 4 * ZROW_THREADS * ZROW_UNROLL) {
    float4 z[ZROW_UNROLL];
#pragma unroll
    for (int u = 0; u < ZROW_UNROLL; ++u) {
      const int v = v0 + u * 4 * ZROW_THREADS;
      z[u] = (counts && v < V) ? *reinterpret_cast<const float4*>(zr + v)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < ZROW_UNROLL; ++u) {
      const int v = v0 + u * 4 * ZROW_THREADS;
      if (v >= vend) break;
      float q[4] = {0.f, 0.f, 0.f, 0.f};
      if (counts && v < V) {
        const float zz[4] = {z[u].x, z[u].y, z[u].z, z[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          q[j] = (v + j < V) ? ex2_approx(fmaf(zz[j], LOG2E, -lse2)) : 0.f;
      }
      uint2 o;
      o.x = pack_bf16x2(q[0], q[1]);
      o.y = pack_bf16x2(q[2], q[3]);
      *reinterpret_cast<uint2*>(dz + ((static_cast<int64_t>(v >> 6) * cap + dr) << 6) + (v & 63)) = o;
    }
  }
  __syncthreads();
  // teacher entries: the first of each run of equal ids rewrites its column
  // (q minus every p of the run, subtracted in sorted order)
  if (counts) {
    const int2* pr = pairs + t * K;
    for (int k = threadIdx.x; k < K; k += ZROW_THREADS) {
      const int id = pr[k].x;
      if (id < 0 || id >= V || (k > 0 && pr[k - 1].x == id)) continue;
      float x = ex2_approx(fmaf(zr[id], LOG2E, -lse2));
      for (int j = k; j < K && pr[j].x == id; ++j) x -= __int_as_float(pr[j].y);
      const uint32_t b = pack_bf16x2(x, 0.f);
      dz[((static_cast<int64_t>(id >> 6) * cap + dr) << 6) + (id & 63)] = static_cast<uint16_t>(b & 0xFFFFu);
    }
  }
}

// dH (bf16, round to nearest even) from the fp32 sum of its vocabulary slabs.
__global__ void __launch_bounds__(256)
dh_convert_kernel(const float4* __restrict__ src, int64_t n4, uint2* __restrict__ dst) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = src[i];
    dst[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

// loss = (sum of the rows' terms, in a fixed order, in fp64) / N.
constexpr int ROWSUM_THREADS = 1024;

__global__ void __launch_bounds__(ROWSUM_THREADS)
rowsum_loss_kernel(const float* __restrict__ rowloss, int64_t T, const int* countN, float* loss,
                   double* numer) {
  __shared__ double s[ROWSUM_THREADS];
  double v = 0.0;
  for (int64_t t = threadIdx.x; t < T; t += ROWSUM_THREADS) v += static_cast<double>(rowloss[t]);
  s[threadIdx.x] = v;
  __syncthreads();
  for (int h = ROWSUM_THREADS / 2; h > 0; h >>= 1) {
    if (threadIdx.x < h) s[threadIdx.x] += s[threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int n = *countN;
    *loss = (n > 0) ? static_cast<float>(s[0] / static_cast<double>(n)) : 0.f;
    *numer = s[0];
  }
}

// ------------------------------------------------------------------ tc GEMM

// dW units of this slot when each slot takes a contiguous range: sized so
// that every slot's total k-block count (its round-robin dH units plus its
// dW units) is near equal.
__device__ __forceinline__ void dw_range(const TcParams& p, int cta, int G, int& b, int& e) {
  const int64_t c6e = p.c6 + 1;  // +1: the dW epilogue is not free
  const int64_t total = static_cast<int64_t>(p.n5) * p.c5 + static_cast<int64_t>(p.n6) * c6e;
  const int64_t target = (total + G - 1) / G;
  int64_t P = 0, Pc = 0, mine = 0;
  for (int j = 0; j < G; ++j) {
    const int64_t cnt5 = (p.n5 > j) ? (p.n5 - j + G - 1) / G : 0;
    int64_t cap = target - cnt5 * p.c5;
    cap = cap > 0 ? cap : 0;
    if (j < cta) Pc += cap;
    if (j == cta) mine = cap;
    P += cap;
  }
  if (P == 0) {
    b = static_cast<int>(static_cast<int64_t>(p.n6) * cta / G);
    e = static_cast<int>(static_cast<int64_t>(p.n6) * (cta + 1) / G);
  } else {
    b = static_cast<int>(static_cast<int64_t>(p.n6) * Pc / P);
    e = static_cast<int>(static_cast<int64_t>(p.n6) * (Pc + mine) / P);
  }
}

// Walks this CTA's work in the order every role sees it.  One "job" is one
// accumulator tile: FWD / DZ: (unit, vocabulary tile); DHDW: one unit.
struct JobIter {
  int mode, G, cta;  // G scheduling slots (CTAs, or CTA pairs); this slot
  // FWD: unit u = (row block u % n_rb, split u / n_rb) over tiles [vt, vt_hi).
  // DZ: tiles dealt round-robin in vocabulary-major order (tile lin = vt n_rb
  // + rb), so that the slots work on neighbouring tiles at any time and share
  // their W tile and H rows in L2; u = the tile's row block.
  // DHDW: dH units round-robin (u = row block x n_nt + d tile), then dW tiles
  // (u = vocabulary block x n_nt + d tile), either as a contiguous range per
  // slot (dw_mode 0: a slot's consecutive tiles share their dZ panels) or
  // dealt in rounds (dw_mode 1): in round k every slot whose quota exceeds k
  // takes the next tile, so the tiles in flight are neighbours and share dZ
  // panels and H_c^T in L2 when one slot's panels alone would not stay there.
  // Round quotas come in two classes: the r5 = n5 mod G slots with one more
  // dH unit hold Qh tiles (the first Eh of them) or Qh - 1, the others Ql
  // (the first El of them) or Ql - 1; the tile index is then closed-form.
  int u, vt, vt_hi;
  int lin;
  int phase;  // DHDW: 0 = dH units, 1 = dW tiles, 2 = done
  int k6, e6;
  int ord;  // jobs of this slot before this one
  // tiles of a class (n slots, quota Q for the first E, Q - 1 for the rest)
  // dealt in rounds before round k, and those of its first m slots in round k
  __device__ static int cls_before(int k, int n, int Q, int E) {
    if (Q < 1) return 0;
    return (k < Q - 1 ? k : Q - 1) * n + (k > Q - 1 ? E : 0);
  }
  __device__ static int cls_rank(int k, int m, int Q, int E) {
    if (Q < 1 || k > Q - 1) return 0;
    return (k < Q - 1) ? m : (m < E ? m : E);
  }
  // DHDW: the next dW tile of this slot (k6 counts them), or phase 2
  __device__ void dw_pick(const TcParams& p) {
    if (p.dw_mode == 0) {
      if (k6 >= e6) { phase = 2; return; }
      u = k6;
      return;
    }
    const int r5 = p.n5 % G;
    const int nl = G - r5;
    const bool heavy = cta < r5;
    const int q = heavy ? p.dw_Qh - 1 + (cta < p.dw_Eh ? 1 : 0)
                        : p.dw_Ql - 1 + (cta - r5 < p.dw_El ? 1 : 0);
    if (k6 >= q) { phase = 2; return; }
    u = cls_before(k6, r5, p.dw_Qh, p.dw_Eh) + cls_before(k6, nl, p.dw_Ql, p.dw_El) +
        cls_rank(k6, cta < r5 ? cta : r5, p.dw_Qh, p.dw_Eh) +
        (cta > r5 ? cls_rank(k6, cta - r5, p.dw_Ql, p.dw_El) : 0);
  }
  // FWD unit -> (row block, split).  Row-block-fastest by default: the units
  // in flight sweep the same W tiles of a split, and every row block's H
  // stays in L2.  When all of H does not fit there (split_fast), split-
  // fastest: the units in flight hold about G / S row blocks and S W tiles.
  // (DZ: u is the row block itself.)
  __device__ int unit_rb(const TcParams& p, int unit) const {
    return (mode != MODE_DZ && p.split_fast) ? unit / p.S : unit % p.n_rb;
  }
  __device__ int unit_s(const TcParams& p, int unit) const {
    return p.split_fast ? unit % p.S : unit / p.n_rb;
  }
  __device__ void vt_range(const TcParams& p, int unit, int& lo, int& hi) const {
    const int s = unit_s(p, unit);
    lo = static_cast<int>(static_cast<int64_t>(s) * p.n_vt / p.S);
    hi = static_cast<int>(static_cast<int64_t>(s + 1) * p.n_vt / p.S);
  }
  __device__ void init(const TcParams& p, int mode_, int per_slot) {
    mode = mode_;
    ord = 0;
    G = gridDim.x / per_slot;
    cta = blockIdx.x / per_slot;
    if (mode == MODE_DZ) {
      lin = cta;
      u = lin % p.n_rb;
      vt = lin / p.n_rb;
      vt_hi = vt + 1;
    } else if (mode != MODE_DHDW) {
      u = cta;
      vt = vt_hi = 0;
      if (u < p.n_units) vt_range(p, u, vt, vt_hi);
    } else {
      u = cta;
      phase = 0;
      if (u >= p.n5) {
        phase = 1;
        dw_start(p);
      }
    }
  }
  __device__ bool valid(const TcParams& p) const {
    if (mode == MODE_DZ) return lin < p.n_units;
    return (mode != MODE_DHDW) ? (u < p.n_units) : (phase < 2);
  }
  // DHDW: sweep this job's k-blocks backwards?  A slot's consecutive jobs
  // alternate direction, so that a job starts on the operand rows the slot's
  // (and, in step, the other slots') previous jobs read last, which L2 still
  // holds: the slab's W rows for the dH units, H_c^T and dZ panels for the
  // dW tiles.
  __device__ bool reverse_k() const { return CKL_SERPENTINE && mode == MODE_DHDW && (ord & 1); }
  __device__ void next(const TcParams& p) {
    ++ord;
    if (mode == MODE_DZ) {
      lin += G;
      u = lin % p.n_rb;
      vt = lin / p.n_rb;
      vt_hi = vt + 1;
    } else if (mode != MODE_DHDW) {
      if (++vt >= vt_hi) {
        u += G;
        if (u < p.n_units) vt_range(p, u, vt, vt_hi);
      }
    } else if (phase == 0) {
      u += G;
      if (u >= p.n5) {
        phase = 1;
        dw_start(p);
      }
    } else {
      ++k6;
      dw_pick(p);
    }
  }
  __device__ void dw_start(const TcParams& p) {
    if (p.dw_mode == 0) {
      dw_range(p, cta, G, k6, e6);
    } else {
      k6 = 0;
    }
    dw_pick(p);
  }
  // FWD / DZ: is this the first / last tile of its unit?  (DZ: every tile
  // starts its row state afresh.)
  __device__ bool first_of_unit(const TcParams& p) const {
    if (mode == MODE_DZ) return true;
    int lo, hi;
    vt_range(p, u, lo, hi);
    return vt == lo;
  }
  __device__ bool last_of_unit() const { return vt + 1 == vt_hi; }
};

// F32: fp32 operands on kind::tf32 MMAs.  A 128-byte swizzle row holds 64
// bf16 or 32 fp32 elements, so a stage carries K = 64 or 32 in the same
// bytes, and an MMA takes K = 16 or 8: four MMAs per stage either way, the
// same shared-memory layout, the same cycles per stage.
template <int MODE, bool PAIR, bool F32 = false>
__global__ void __launch_bounds__(Cfg<MODE, PAIR>::THREADS, 1)
tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<MODE, PAIR>;
  constexpr int KE = F32 ? 32 : 64;               // K elements per stage (one 128-byte row)
  constexpr int KI = F32 ? 8 : 16;                // K per MMA instruction
  constexpr uint32_t ATOM_B = 128u * KE;          // one MN-major atom column: KE x KE elements
  constexpr uint32_t MN_STEP = 128u * KI;         // MN-major descriptor advance per MMA
  // MN-major operands: bf16 in the 128-byte swizzle (8-row atoms, SBO 1024);
  // tf32 in the 128-byte / 32-byte-base swizzle (4-row atoms, SBO 512)
  constexpr uint32_t MN_SBO = F32 ? 512u : 1024u;
  constexpr int STAGES = C::STAGES;
  constexpr int EPI_WARPS = C::EPI_WARPS;
  constexpr int B_STAGE = C::B_STAGE;
  constexpr int MB = C::MB;
  constexpr uint32_t MMA_M = PAIR ? 2 * BM : BM;
  extern __shared__ uint8_t smem_raw[];
  // 1 KB-aligned base for the 128-byte swizzled tiles.  Both CTAs of a pair
  // get the same layout, so every offset names the same slot in either CTA.
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = the pair's leader
  const bool leader = (rank == 0);
  const uint32_t bar_full = sbase + C::BAR_OFF;               // [STAGES] (leader's count both)
  const uint32_t bar_empty = bar_full + 8 * STAGES;           // [STAGES]
  const uint32_t bar_tfull = bar_empty + 8 * STAGES;          // [2]
  const uint32_t bar_tempty = bar_tfull + 16;                 // [2] (leader's count both)
  const uint32_t bar_drain = bar_tempty + 16;                 // [1]
  const uint32_t bar_staged = bar_drain + 8;                  // [2] staging tile written
  const uint32_t bar_sfree = bar_staged + 16;                 // [2] staging tile read out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::BAR_OFF + 8 * (2 * STAGES + 9));

  if (warp == 0 && lane == 0) {
    const int n_maps = (MODE == MODE_FWD) ? 2 : (MODE == MODE_DHDW) ? 6 : 3;
#pragma unroll 1
    for (int i = 0; i < n_maps; ++i) prefetch_tmap(&p.tm[i]);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, PAIR ? 2 : 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_tfull + 8 * a, 1);
      mbar_init(bar_tempty + 8 * a, (PAIR ? 2 : 1) * 32 * EPI_WARPS);
    }
    mbar_init(bar_drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_staged + 8 * b, EPI_WARPS);
      mbar_init(bar_sfree + 8 * b, 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();  // the peer may signal the leader's barriers from here on
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  // The backward's GEMMs are launched so that the next one may start while
  // this one finishes (its CTAs take the SMs this one's CTAs leave): allow
  // that now.  Whatever reads or writes memory that an earlier launch of the
  // stream writes or reads waits below for that launch (griddep_wait), and
  // only after that: the dH / dW producer before its first dZ load, every
  // epilogue before its first global access.  The logit GEMMs' producers read
  // H and W alone, so a recompute launch computes its first tiles while the
  // dH / dW launch ahead of it drains.
  griddep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      if (MODE == MODE_DHDW) griddep_wait();  // dZ, H_c^T: written by the launches ahead
      JobIter it;
      it.init(p, MODE, PAIR ? 2 : 1);
      for (; ok && it.valid(p); it.next(p)) {
        int nkb;
        int a_x = 0, a_y = 0, b_x = 0, b_y = 0, kind = 0;
        const int half_n = PAIR ? p.bn / 2 : p.bn;  // B rows / columns this CTA stages
        if (MODE != MODE_DHDW) {
          const int rb = it.unit_rb(p, it.u);
          nkb = (p.d + KE - 1) / KE;
          a_y = rb * MB + static_cast<int>(rank) * BM;
          b_y = (p.vt0 + it.vt) * BN_V + static_cast<int>(rank) * (BN_V / (PAIR ? 2 : 1));
        } else if (it.phase == 0) {
          kind = 5;
          nkb = p.c5;
          a_y = (it.u / p.n_nt) * MB + static_cast<int>(rank) * BM;      // chunk rows
          b_x = (it.u % p.n_nt) * p.bn + static_cast<int>(rank) * half_n;  // d offset
        } else {
          kind = 6;
          nkb = p.c6;
          a_x = (it.u / p.n_nt) * MB + static_cast<int>(rank) * BM;      // vocabulary rows
          b_x = (it.u % p.n_nt) * p.bn + static_cast<int>(rank) * half_n;
        }
        const uint32_t bytes = (MODE != MODE_DHDW) ? A_BYTES + B_STAGE : A_BYTES + half_n * 128;
        const bool rev = it.reverse_k();
        for (int kq = 0; kq < nkb; ++kq) {
          const int kb = rev ? nkb - 1 - kq : kq;  // the k-block this stage carries
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1u, p.status)) { ok = false; break; }
          uint32_t fb = bar_full + 8 * stage;
          if (PAIR) {
            // The leader's barrier counts both CTAs' bytes; the peer arrives on it.
            if (leader) mbar_arrive_expect_tx(fb, 2 * bytes);
            fb = mapa_shared(fb, 0);
            if (!leader) mbar_arrive_cluster(fb);
          } else {
            mbar_arrive_expect_tx(fb, bytes);
          }
          const uint32_t sa = sbase + C::A_OFF + stage * A_BYTES;
          const uint32_t sb = sbase + C::B_OFF + stage * B_STAGE;
          if (MODE != MODE_DHDW) {
            if (PAIR) {
              tma_load_2d_pair(sa, &p.tm[0], fb, kb * KE, a_y);
              tma_load_2d_pair(sb, &p.tm[1], fb, kb * KE, b_y);
            } else {
              tma_load_2d(sa, &p.tm[0], fb, kb * KE, a_y);
              tma_load_2d(sb, &p.tm[1], fb, kb * KE, b_y);
            }
          } else if (kind == 5) {
            // dZ is stored as 64-column panels: k-block kb is panel kb.  W is
            // MN-major here: one 64-column atom per box.
            if (PAIR) {
              tma_load_3d_pair(sa, &p.tm[0], fb, 0, a_y, kb);
              if (p.w3d) {
                // W viewed as [d / KE][V][KE]: this CTA's half_n columns are
                // half_n / KE atoms, one box, landing ATOM_B apart
                tma_load_3d_pair(sb, &p.tm[1], fb, 0, p.v_lo + kb * KE, b_x / KE);
              } else {
                for (int j = 0; j < half_n / KE; ++j)
                  tma_load_2d_pair(sb + j * ATOM_B, &p.tm[1], fb, b_x + KE * j,
                                   p.v_lo + kb * KE);
              }
            } else {
              tma_load_3d(sa, &p.tm[0], fb, 0, a_y, kb);
              for (int j = 0; j < half_n / KE; ++j)
                tma_load_2d(sb + j * ATOM_B, &p.tm[1], fb, b_x + KE * j, p.v_lo + kb * KE);
            }
          } else {
            // A = dZ^T: one box holding the two 64-column panels of this
            // vocabulary row block (8 KB each, one MN-major atom column each).
            // B = H_c^T (d rows x chunk rows, chunk rows contiguous): K-major.
            if (PAIR) {
              tma_load_3d_pair(sa, &p.tm[2], fb, 0, kb * KE, a_x / KE);
              tma_load_2d_pair(sb, &p.tm[3], fb, kb * KE, b_x);
            } else {
              tma_load_3d(sa, &p.tm[2], fb, 0, kb * KE, a_x / KE);
              tma_load_2d(sb, &p.tm[3], fb, kb * KE, b_x);
            }
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Let every load this thread started land before the CTA can exit.  A
      // pair's loads all count on the leader's barriers, so the leader waits.
      if (leader) {
        for (int s = 0; s < STAGES; ++s) {
          if (issued > static_cast<uint32_t>(s)) {
            const uint32_t last = issued - 1 - ((issued - 1 - s) % STAGES);
            mbar_wait(bar_full + 8 * s, (last / STAGES) & 1u, p.status);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // (the leader's; a pair's peer only holds its TMEM)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      JobIter it;
      it.init(p, MODE, PAIR ? 2 : 1);
      for (; ok && it.valid(p); it.next(p)) {
        int nkb;
        uint32_t idesc;
        uint32_t a_step, b_step, a_lbo, b_lbo;
        bool a_mn = false, b_mn = false;
        if (MODE != MODE_DHDW) {
          nkb = (p.d + KE - 1) / KE;
          idesc = F32 ? idesc_tf32(MMA_M, BN_V, 0, 0) : idesc_bf16(MMA_M, BN_V, 0, 0);
          a_step = 32; b_step = 32; a_lbo = 16; b_lbo = 16;
        } else if (it.phase == 0) {
          nkb = p.c5;
          idesc = F32 ? idesc_tf32(MMA_M, p.bn, 0, 1) : idesc_bf16(MMA_M, p.bn, 0, 1);
          a_step = 32; b_step = MN_STEP; a_lbo = 16; b_lbo = ATOM_B;
          b_mn = true;
        } else {
          nkb = p.c6;
          idesc = F32 ? idesc_tf32(MMA_M, p.bn, 1, 0) : idesc_bf16(MMA_M, p.bn, 1, 0);
          a_step = MN_STEP; b_step = 32; a_lbo = ATOM_B; b_lbo = 16;
          a_mn = true;
        }
        if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1u, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * ACC_COLS;
        // descriptors of stage 0's operands for this job (a_mn / b_mn: that
        // operand is MN-major, dH's W or dW's dZ^T); a stage, or a K step
        // within it, only moves the start address, the low 14 bits in
        // 16-byte units, which stay below 2^14 for any shared-memory address
        const uint64_t ad0 = (F32 && a_mn) ? sdesc_sw128_b32(sbase + C::A_OFF, a_lbo, MN_SBO)
                                           : sdesc_sw128(sbase + C::A_OFF, a_lbo, 1024);
        const uint64_t bd0 = (F32 && b_mn) ? sdesc_sw128_b32(sbase + C::B_OFF, b_lbo, MN_SBO)
                                           : sdesc_sw128(sbase + C::B_OFF, b_lbo, 1024);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(bar_full + 8 * stage, phase, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ads = ad0 + static_cast<uint64_t>((stage * A_BYTES) >> 4);
          const uint64_t bds = bd0 + static_cast<uint64_t>((stage * B_STAGE) >> 4);
#pragma unroll
          for (int kk = 0; kk < KE / KI; ++kk) {
            const uint64_t ad = ads + static_cast<uint64_t>((kk * a_step) >> 4);
            const uint64_t bd = bds + static_cast<uint64_t>((kk * b_step) >> 4);
            const uint32_t acc_in = (kb | kk) != 0 ? 1u : 0u;
            if constexpr (F32) {
              if (PAIR) umma_tf32_pair(d_tmem, ad, bd, idesc, acc_in);
              else umma_tf32(d_tmem, ad, bd, idesc, acc_in);
            } else {
              if (PAIR) umma_bf16_pair(d_tmem, ad, bd, idesc, acc_in);
              else umma_bf16(d_tmem, ad, bd, idesc, acc_in);
            }
          }
          if (PAIR) umma_commit_pair(bar_empty + 8 * stage, 3);
          else umma_commit(bar_empty + 8 * stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (PAIR) umma_commit_pair(bar_tfull + 8 * acc, 3);
        else umma_commit(bar_tfull + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // Every MMA this thread issued has finished before TMEM is released.
      if (PAIR) umma_commit_pair(bar_drain, 1);
      else umma_commit(bar_drain);
      mbar_wait(bar_drain, 0, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0 .. EPI_WARPS-1
    const int lg = warp & 3;                 // TMEM lane group this warp may access
    static_assert(EPI_WARPS == 4, "one warp per TMEM lane group");
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    const int row_in_tile = static_cast<int>(rank) * BM + lg * 32 + lane;  // within MB
    const int row0_cta = static_cast<int>(rank) * BM;  // this CTA's rows within MB
    // Stores go through two alternating 128-row staging tiles: every warp
    // writes its 32 rows, and one thread stores the whole tile with a single
    // TMA call once all four warps have arrived (4x fewer TMA operations than
    // a store per warp; the TMA unit is shared with the operand loads).
    const uint32_t stage_base = sbase + C::EPI_OFF;
    const uint32_t srow = static_cast<uint32_t>(lg * 32 + lane);  // staging row of this thread
    const bool issuer = (ew == 0 && lane == 0);
    const uint32_t tempty_leader = PAIR ? mapa_shared(bar_tempty, 0) : bar_tempty;
    int acc = 0;
    uint32_t acc_phase = 0;
    int nstore = 0;
    bool ok = true;
    // Wait until staging tile nstore & 1 has been read out by its previous store.
    auto stage_begin = [&]() -> bool {
      bool good = true;
      if (lane == 0 && nstore >= 2)
        good = mbar_wait(bar_sfree + 8 * (nstore & 1), static_cast<uint32_t>((nstore >> 1) - 1) & 1u,
                         p.status);
      __syncwarp();
      return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    };
    // Publish this warp's rows; the issuer stores the tile once all warps have
    // (kind 0: dZ panel, 1: dH, 2: dW store, 3: dW add, 4: logits, 5: fp32 dH
    // store, 6: fp32 dH add) and then frees the
    // tile of the store before.
    auto stage_end = [&](int kind, int x, int y, int z) -> bool {
      fence_proxy_async_smem();
      __syncwarp();
      const uint32_t sb = static_cast<uint32_t>(nstore & 1);
      if (lane == 0) mbar_arrive(bar_staged + 8 * sb);
      bool good = true;
      if (issuer) {
        good = mbar_wait(bar_staged + 8 * sb, static_cast<uint32_t>(nstore >> 1) & 1u, p.status);
        if (good) {
          const uint32_t buf = stage_base + sb * EPI_STAGE;
          if (kind == 0) tma_store_3d(&p.tm[2], buf, x, y, z);
          else if (kind == 1) tma_store_2d(&p.tm[4], buf, x, y);
          else if (kind == 2) tma_store_2d(&p.tm[5], buf, x, y);
          else if (kind == 3) tma_reduce_add_2d(&p.tm[5], buf, x, y);
          else if (kind == 4) tma_store_2d(&p.tm[2], buf, x, y);
          else if (kind == 5) tma_store_2d(&p.tm[4], buf, x, y);
          else tma_reduce_add_2d(&p.tm[4], buf, x, y);
          bulk_commit();
          if (nstore >= 1) {
            bulk_wait_read<1>();
            mbar_arrive(bar_sfree + 8 * (sb ^ 1u));
          }
        }
      }
      ++nstore;
      return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    };

    // per-row state (FWD / DZ)
    int64_t t = 0;
    bool row_ok = false, counts = false;
    int cur = 0;
    int nidx = INT_MAX;
    float np_ = 0.f;
    float run_m = -INFINITY, run_s = 0.f, run_pz = 0.f;
    float lse2 = 0.f;
    float scale = 0.f;
    griddep_wait();  // every epilogue reads or writes what earlier launches touch
    if (MODE == MODE_DHDW) {
      const int n = *p.countN;
      const float g = (p.grad_loss != nullptr) ? *p.grad_loss : 1.f;
      scale = (n > 0) ? g / static_cast<float>(n) : 0.f;
    }

    JobIter it;
    it.init(p, MODE, PAIR ? 2 : 1);
    for (; ok && it.valid(p); it.next(p)) {
      if (MODE != MODE_DHDW && it.first_of_unit(p)) {
        const int rb = it.unit_rb(p, it.u);
        const int r = rb * MB + row_in_tile;  // row within T (FWD) or the chunk (DZ)
        row_ok = r < p.rows;
        t = static_cast<int64_t>(p.row0) + r;
        counts = row_ok && (p.mask == nullptr || p.mask[t] != 0);
        run_m = -INFINITY; run_s = 0.f; run_pz = 0.f;
        nidx = INT_MAX;
        if (MODE == MODE_DZ && row_ok) lse2 = p.lse[t] * LOG2E;
        const bool want_ids = (MODE == MODE_DZ) ? counts : row_ok;
        if (want_ids) {
          const int2* pr = p.pairs + t * p.K;
          const int v_lo = p.v_off + (p.vt0 + it.vt) * BN_V;
          int lo = 0, hi = p.K;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (pr[mid].x < v_lo) lo = mid + 1; else hi = mid;
          }
          cur = lo;
          if (cur < p.K) { const int2 e = pr[cur]; nidx = e.x; np_ = __int_as_float(e.y); }
        }
      }
      if (!mbar_wait(bar_tfull + 8 * acc, acc_phase, p.status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tacc = tmem_base + lane_off + static_cast<uint32_t>(acc) * ACC_COLS;

      if (MODE == MODE_FWD || MODE == MODE_FWDZ) {
        const int zy0 = it.unit_rb(p, it.u) * MB + row0_cta;  // FWDZ: first chunk row of this CTA
        for (int c = 0; c < BN_V / 32; ++c) {
          const int v0 = (p.vt0 + it.vt) * BN_V + c * 32;
          if (v0 >= p.V) break;
          float x[32];
          tmem_ld32(tacc + c * 32, x);
          if (MODE == MODE_FWDZ) {
            // the fp32 logits of this 128 x 32 block (columns past V are clipped by the store)
            if (!stage_begin()) { ok = false; break; }
            const uint32_t rowa = stage_base + (nstore & 1) * EPI_STAGE + srow * 128;
            const int sw = lane & 7;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_v4(rowa + ((j ^ sw) << 4), __float_as_uint(x[4 * j]),
                           __float_as_uint(x[4 * j + 1]), __float_as_uint(x[4 * j + 2]),
                           __float_as_uint(x[4 * j + 3]));
            if (!stage_end(4, v0, zy0, 0)) { ok = false; break; }
          }
          if (v0 + 32 > p.V) {
#pragma unroll
            for (int j = 0; j < 32; ++j) if (v0 + j >= p.V) x[j] = -INFINITY;
          }
          float cm = x[0];
#pragma unroll
          for (int j = 1; j < 32; ++j) cm = fmaxf(cm, x[j]);
          const float ym = cm * LOG2E;
          if (ym > run_m) { run_s *= ex2_approx(run_m - ym); run_m = ym; }
          float se = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) se += ex2_approx(fmaf(x[j], LOG2E, -run_m));
          run_s += se;
          // ids past this launch's last column (another vocabulary shard's) stop the walk
          const int v_hi = p.v_off + min(v0 + 32, p.V);
          while (nidx < v_hi) {
            const int off = nidx - p.v_off - v0;
            float val = x[0];
#pragma unroll
            for (int j = 1; j < 32; ++j) val = (off == j) ? x[j] : val;
            run_pz = fmaf(np_, val, run_pz);
            ++cur;
            if (cur < p.K) { const int2 e = p.pairs[t * p.K + cur]; nidx = e.x; np_ = __int_as_float(e.y); }
            else nidx = INT_MAX;
          }
        }
      } else if (MODE == MODE_DZ) {
        const int rb = it.u % p.n_rb;
        const int y0 = rb * MB + row0_cta;  // first chunk row of this CTA's 128
        const int v_end = (p.V + 63) & ~63;  // dZ panels span round_up(V, 64) columns
        for (int c = 0; c < BN_V / 32; ++c) {
          const int v0 = (p.vt0 + it.vt) * BN_V + c * 32;
          if (v0 >= v_end) break;
          float x[32];
          tmem_ld32(tacc + c * 32, x);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            x[j] = counts ? ex2_approx(fmaf(x[j], LOG2E, -lse2)) : 0.f;
          const int v_hi = p.v_off + min(v0 + 32, p.V);
          while (nidx < v_hi) {
            const int off = nidx - p.v_off - v0;
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] -= (off == j) ? np_ : 0.f;
            ++cur;
            if (cur < p.K) { const int2 e = p.pairs[t * p.K + cur]; nidx = e.x; np_ = __int_as_float(e.y); }
            else nidx = INT_MAX;
          }
          if (v0 + 32 > p.V) {
            // the last panel's columns past V are read by the dH GEMM: write 0 there
#pragma unroll
            for (int j = 0; j < 32; ++j) if (v0 + j >= p.V) x[j] = 0.f;
          }
          if (!stage_begin()) { ok = false; break; }
          if constexpr (F32) {
            // fp32 panels are 32 columns wide: this chunk is one whole panel.
            // 128-byte rows, 128-byte swizzle: unit j of row r at unit j ^ (r & 7)
            const uint32_t rowa = stage_base + (nstore & 1) * EPI_STAGE + srow * 128;
            const int sw = lane & 7;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_v4(rowa + ((j ^ sw) << 4), __float_as_uint(x[4 * j]),
                           __float_as_uint(x[4 * j + 1]), __float_as_uint(x[4 * j + 2]),
                           __float_as_uint(x[4 * j + 3]));
            if (!stage_end(0, 0, y0, (v0 - p.vt0 * BN_V) >> 5)) { ok = false; break; }
          } else {
            // 64-byte rows, 64-byte swizzle: 16-byte unit j of row r at unit j ^ ((r >> 1) & 3)
            const uint32_t rowa = stage_base + (nstore & 1) * EPI_STAGE + srow * 64;
            const int sw = (lane >> 1) & 3;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(rowa + ((j ^ sw) << 4), pack_bf16x2(x[8 * j], x[8 * j + 1]),
                           pack_bf16x2(x[8 * j + 2], x[8 * j + 3]),
                           pack_bf16x2(x[8 * j + 4], x[8 * j + 5]),
                           pack_bf16x2(x[8 * j + 6], x[8 * j + 7]));
            // panel of this slab's buffer
            if (!stage_end(0, v0 & 63, y0, (v0 - p.vt0 * BN_V) >> 6)) { ok = false; break; }
          }
        }
      } else {
        // DHDW: scale and write one accumulator tile (this CTA's rows, all columns).
        const bool is_dh = (it.phase == 0);
        const int nt = it.u % p.n_nt;
        // dH: rows of the row chunk; dW: vocabulary rows (the slab starts at v_lo)
        const int y0 = (it.u / p.n_nt) * MB + row0_cta + (is_dh ? 0 : p.v_lo);
        const bool bf16_out = is_dh && p.dh_mode == 0;
        for (int c = 0; c < p.bn / 32; ++c) {
          const int x0 = nt * p.bn + c * 32;
          if (x0 >= p.d) break;
          float x[32];
          tmem_ld32(tacc + c * 32, x);
          if (!stage_begin()) { ok = false; break; }
          const uint32_t buf = stage_base + (nstore & 1) * EPI_STAGE;
          if (bf16_out) {
            const uint32_t rowa = buf + srow * 64;
            const int sw = (lane >> 1) & 3;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(rowa + ((j ^ sw) << 4), pack_bf16x2(x[8 * j] * scale, x[8 * j + 1] * scale),
                           pack_bf16x2(x[8 * j + 2] * scale, x[8 * j + 3] * scale),
                           pack_bf16x2(x[8 * j + 4] * scale, x[8 * j + 5] * scale),
                           pack_bf16x2(x[8 * j + 6] * scale, x[8 * j + 7] * scale));
          } else {
            // 128-byte rows, 128-byte swizzle: unit j of row r at unit j ^ (r & 7)
            const uint32_t rowa = buf + srow * 128;
            const int sw = lane & 7;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_v4(rowa + ((j ^ sw) << 4), __float_as_uint(x[4 * j] * scale),
                           __float_as_uint(x[4 * j + 1] * scale),
                           __float_as_uint(x[4 * j + 2] * scale),
                           __float_as_uint(x[4 * j + 3] * scale));
          }
          const int kind = is_dh ? (p.dh_mode == 0 ? 1 : p.dh_mode == 1 ? 5 : 6)
                                 : (p.dw_store ? 2 : 3);
          if (!stage_end(kind, x0, y0, 0)) { ok = false; break; }
        }
      }
      tc_fence_before();
      if (PAIR) mbar_arrive_cluster(tempty_leader + 8 * acc);
      else mbar_arrive(bar_tempty + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }

      if ((MODE == MODE_FWD || MODE == MODE_FWDZ) && it.last_of_unit() && row_ok) {
        const int s = it.unit_s(p, it.u);
        p.partials[t * p.S + s] = make_float4(run_m, run_s, run_pz, 0.f);
      }
    }
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();  // neither CTA frees TMEM or exits while the pair's MMAs run
  tc_fence_after();
  if (warp == 1) {
    if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace ckl
