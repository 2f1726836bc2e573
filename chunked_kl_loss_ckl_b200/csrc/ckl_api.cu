// Host side of libckl.so: argument checks, workspace layout, the chunk
// scheduler and the kernel launches.  See include/ckl.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/ckl.h"
#include "ckl_kernels.cuh"
#include "ckl_topk.cuh"

namespace {

using ckl::TcParams;

constexpr int32_t kVersion = 100;  // 0.1.0
constexpr int kMaxSplits = 64;     // vocabulary splits per row in the forward
constexpr size_t kHeaderBytes = 256;

// Header words at the start of the workspace.
struct Header {
  int32_t status;   // CKL_DEV_* bits
  int32_t countN;   // positions that count
  uint32_t ticket;  // combine: blocks finished
  uint32_t pad;
  double numer;     // sum over the positions that count of KL_t (fp64), written with the loss
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Blocking of the backward: row chunks of Cr rows x vocabulary slabs of Sv
// columns (n slabs), every block's dZ fitting the chunk x V buffer.
struct Plan {
  int64_t Cr, Sv, n;
};

struct Layout {
  size_t pairs, hp, partials, blocksums, dz, hct, dh32, z, rowloss, total;
  int64_t npanels;  // dZ panels of 64 vocabulary columns (row-chunked schedule)
  int64_t cap;      // rows of one chunk: min(chunk, T)
  int64_t cr_alloc; // rows the sliced schedule may hold (0 = never sliced)
  int64_t pitch_t;  // H_c^T row pitch (elements): max(cap, cr_alloc) rounded up to 8
  int64_t zpitch;   // single pass: fp32 logit row pitch (elements), V rounded up to 4
  int64_t sp_rows;  // single pass: dZ rows held (the chunks of one dH/dW launch)
  int eb;           // bytes per H / W / dZ element: 2 (bf16) or 4 (fp32, tf32 MMAs)
};

// The rows of a sliced block: the Cr that balances the two fp32 accumulations'
// traffic (dW re-added once per row chunk, partial dH once per slab) under
// Cr x Sv = chunk x V, i.e. sqrt(chunk x V), rounded up to 256; but no more
// than keeps H_c^T (Cr x d bf16, which every round of dW tiles streams) within
// 48 MiB of the 126 MB L2.  eb = bytes per element.
int64_t sliced_rows(int64_t T, int64_t d, int64_t V, int64_t cap, int eb) {
  if (T <= cap) return 0;
  int64_t r = static_cast<int64_t>(std::ceil(std::sqrt(static_cast<double>(cap) * V)));
  r = cdiv(r, 256) * 256;
  const int64_t r_l2 = (int64_t(48) << 20) / (eb * d) / 256 * 256;
  r = std::min(r, r_l2);
  return r > cap ? r : 0;
}

// Row-chunked (the pages' schedule: one chunk of rows x all V at a time) or
// sliced (fewer, taller row chunks, each swept in vocabulary slabs), whichever
// moves fewer bytes of fp32 accumulation: row chunking reads and writes dW
// (V x d fp32) once per chunk; slicing writes dW once per tall row chunk and
// reads and writes a partial dH (rows x d fp32) once per slab.
Plan plan_backward(int64_t T, int64_t d, int64_t V, const Layout& L) {
  const int64_t Vp = cdiv(V, 64) * 64;
  const Plan rows_only{L.cap, Vp, 1};
  if (L.cr_alloc == 0) return rows_only;
  const int64_t budget = L.cap * Vp;  // dZ entries the workspace holds
  const int64_t Cr = std::min(T, L.cr_alloc);
  int64_t Sv = budget / Cr / 256 * 256;
  if (Sv < 256 || Sv >= Vp) return rows_only;
  int64_t n = cdiv(Vp, Sv);
  Sv = cdiv(cdiv(Vp, n), 256) * 256;  // even slabs
  n = cdiv(Vp, Sv);
  const double vd4 = 4.0 * static_cast<double>(V) * d, td4 = 4.0 * static_cast<double>(T) * d;
  const double rows_bytes = (2.0 * cdiv(T, L.cap) - 1.0) * vd4;
  const double sliced_bytes = (2.0 * cdiv(T, Cr) - 1.0) * vd4 + (2.0 * n - 1.0) * td4 + 1.5 * td4;
  return sliced_bytes < rows_bytes ? Plan{Cr, Sv, n} : rows_only;
}

// The forward's part of the workspace: header, sorted teacher pairs, sum p log p,
// the vocabulary-split partials (sized for kMaxSplits) and the combine's block
// sums.  Every layout starts with it, at the same offsets.
Layout forward_layout(int64_t T, int32_t K) {
  Layout L{};
  L.eb = 2;
  size_t off = kHeaderBytes;
  L.pairs = off;
  off += align256(static_cast<size_t>(T) * K * 8);
  L.hp = off;
  off += align256(static_cast<size_t>(T) * 4);
  L.partials = off;
  off += align256(static_cast<size_t>(T) * kMaxSplits * 16);
  L.blocksums = off;
  off += align256(static_cast<size_t>(cdiv(T, ckl::COMBINE_THREADS)) * 8);
  L.total = off;
  return L;
}

// Chunks whose dZ the single pass gathers before one dH / dW launch: dW is
// read-modify-written once per group instead of once per chunk.
constexpr int64_t kSpGroup = 4;

// single_pass adds the chunk's fp32 logits [cap][zpitch] and the rows' loss
// terms [T], and holds the dZ of up to kSpGroup chunks.
// eb = 4: the fp32 entry points (dZ and H_c^T in fp32; dH accumulates in the
// caller's fp32 output, so no partial-dH buffer).
Layout layout(int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk, bool single_pass,
              int eb = 2) {
  Layout L = forward_layout(T, K);
  L.eb = eb;
  size_t off = L.total;
  // dZ as 64-column panels: [ceil(V/64)][cap][64] bf16, cap = rows of the
  // largest chunk (a sliced block uses the same bytes as [Sv/64][Cr][64]).
  L.npanels = cdiv(V, 64);
  L.cap = std::min(chunk, std::max<int64_t>(T, 1));
  L.sp_rows = single_pass ? std::min(kSpGroup, cdiv(std::max<int64_t>(T, 1), L.cap)) * L.cap
                          : L.cap;
  L.dz = off;
  off += align256(static_cast<size_t>(L.npanels) * L.sp_rows * 64 * eb);
  // H_c^T for the dW GEMM: [d][pitch_t] bf16.
  L.cr_alloc = sliced_rows(T, d, V, L.cap, eb);
  L.pitch_t = cdiv(std::max(L.sp_rows, L.cr_alloc), 8) * 8;
  L.hct = off;
  off += align256(static_cast<size_t>(d) * L.pitch_t * eb);
  // fp32 dH of a sliced row chunk, summed over its vocabulary slabs.
  L.dh32 = off;
  if (eb == 2) off += align256(static_cast<size_t>(L.cr_alloc) * d * 4);
  L.zpitch = cdiv(V, 4) * 4;
  if (single_pass) {
    L.z = off;
    off += align256(static_cast<size_t>(L.cap) * L.zpitch * 4);
    L.rowloss = off;
    off += align256(static_cast<size_t>(T) * 4);
  }
  L.total = off;
  return L;
}

bool sizes_ok(int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk) {
  const int64_t lim = (int64_t(1) << 31) - 1;
  return T >= 0 && T < lim && d >= 8 && d % 8 == 0 && d < lim && V >= 1 && V < lim && K >= 1 &&
         chunk >= 1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// ---- driver entry point for tensor-map encoding (no link-time libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tiled tensor map over a row-major [outer, inner] array.
bool map2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
           uint64_t outer, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
           CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D tiled tensor map over [d2][d1][d0] with byte pitches p1 (dim 1), p2 (dim 2).
bool map3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
           uint64_t d2, uint64_t p1, uint64_t p2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {p1, p2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map with a box of depth b2 along dim 2 (128-byte swizzle by default).
bool map3d2(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
            uint64_t d2, uint64_t p1, uint64_t p2, uint32_t b0, uint32_t b1, uint32_t b2,
            CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {p1, p2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Every GEMM runs on CTA pairs sharing one cta_group::2 MMA (each CTA
// stages half of the B operand); one scheduling slot = one pair.
constexpr bool kPair = true;
constexpr int kSlotCTAs = kPair ? 2 : 1;
constexpr int64_t kMB = kPair ? 2 * ckl::BM : ckl::BM;  // rows of one job's M extent

struct DevInfo {
  int sms = 0;
  int major = 0;
  bool attrs_set = false;
  int slots[4] = {0, 0, 0, 0};  // co-resident CTA pairs per GEMM mode
};

// Element type of a launch's operands: bf16 (kind::f16) or fp32 (kind::tf32).
template <bool F32>
constexpr CUtensorMapDataType kDT =
    F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
template <bool F32>
constexpr uint32_t kKE = F32 ? 32 : 64;  // K (and panel) elements per 128-byte row

// attr: room for 2.  The backward's GEMMs (DZ, DHDW) may start before the
// launch ahead of them ends (programmatic stream serialisation; the kernel
// waits where it depends on it).
#ifndef CKL_PDL
#define CKL_PDL 1
#endif
template <int MODE>
cudaLaunchConfig_t tc_config(int slots, cudaStream_t st, cudaLaunchAttribute* attr,
                             bool dependent = true) {
  using C = ckl::Cfg<MODE, kPair>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(slots * kSlotCTAs));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_ALLOC;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSlotCTAs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (CKL_PDL && dependent && (MODE == ckl::MODE_DZ || MODE == ckl::MODE_DHDW)) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  }
  return cfg;
}

template <int MODE>
bool setup_mode(DevInfo& di) {
  using C = ckl::Cfg<MODE, kPair>;
  if (cudaFuncSetAttribute(ckl::tc_kernel<MODE, kPair>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) !=
      cudaSuccess)
    return false;
  // the fp32 form has the same shared memory and threads, so the same occupancy
  if constexpr (MODE != ckl::MODE_FWDZ) {
    if (cudaFuncSetAttribute(ckl::tc_kernel<MODE, kPair, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) !=
        cudaSuccess)
      return false;
  }
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = tc_config<MODE>(di.sms / kSlotCTAs, nullptr, attr, false);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, ckl::tc_kernel<MODE, kPair>, &cfg) != cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    n = di.sms / kSlotCTAs;
  }
  di.slots[MODE] = std::min(n, di.sms / kSlotCTAs);
  return true;
}

// Launches one persistent GEMM on min(co-resident slots, units) CTA pairs.
template <int MODE, bool F32 = false>
int launch_tc(const TcParams& p, int64_t units, const DevInfo& di, cudaStream_t st) {
  const int slots = static_cast<int>(std::min<int64_t>(di.slots[MODE], units));
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = tc_config<MODE>(slots, st, attr);
  return cudaLaunchKernelEx(&cfg, ckl::tc_kernel<MODE, kPair, F32>, p) == cudaSuccess
             ? CKL_OK
             : CKL_ERR_CUDA;
}

bool device_info(DevInfo& out) {
  static std::mutex mu;
  static DevInfo cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  DevInfo& di = cache[dev];
  if (di.sms == 0) {
    if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&di.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return false;
  }
  if (!di.attrs_set && di.major == 10) {
    if (!setup_mode<ckl::MODE_FWD>(di) || !setup_mode<ckl::MODE_DZ>(di) ||
        !setup_mode<ckl::MODE_DHDW>(di) || !setup_mode<ckl::MODE_FWDZ>(di))
      return false;
    di.attrs_set = true;
  }
  out = di;
  return true;
}

// Records launch events around one kernel.
struct TraceScope {
  ckl_trace* tr;
  cudaStream_t st;
  int slot = -1;
  TraceScope(ckl_trace* t, cudaStream_t s, int kid) : tr(t), st(s) {
    if (tr && tr->events && tr->count < tr->capacity) {
      slot = tr->count;
      cudaEventRecord(static_cast<cudaEvent_t>(tr->events[2 * slot]), st);
      if (tr->kernel_id) tr->kernel_id[slot] = kid;
    }
  }
  ~TraceScope() {
    if (slot >= 0) {
      cudaEventRecord(static_cast<cudaEvent_t>(tr->events[2 * slot + 1]), st);
      tr->count = slot + 1;
    }
  }
};

// Vocabulary splits S for n_rb row blocks: the most even makespan over the
// SMs (every unit = one row block x one contiguous run of vocabulary tiles),
// with S in [smin, smax].
int choose_splits(int64_t n_rb, int64_t n_vt, int sms, int smin = 1, int smax_in = kMaxSplits) {
  int best = std::max(1, std::min<int>(smin, static_cast<int>(n_vt)));
  double best_cost = 1e300;
  const int smax = static_cast<int>(std::min<int64_t>(std::min(kMaxSplits, smax_in), n_vt));
  for (int S = std::max(1, smin); S <= smax; ++S) {
    const int64_t units = n_rb * S;
    const int64_t waves = cdiv(units, sms);
    const double per_unit = static_cast<double>(cdiv(n_vt, S)) + 0.25;  // +: unit set-up
    const double cost = static_cast<double>(waves) * per_unit;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

// d-tile width of the dH / dW GEMMs.  A narrower tile wastes fewer padded
// columns but reads more shared memory per FLOP: at M = 256 (a CTA pair) and
// N = 128 each MMA needs as many operand bytes per clock as shared memory
// delivers, so those tiles run well below the tensor peak (a d = 2880 head
// measured 690 against 1270 TFLOP/s).  Cost per column: padded width, times
// 1.5 for N = 128 (2 for N = 64).
// Splits and unit order of a forward launch over n_rb row blocks: when the
// row blocks' H (kMB x d each) does not fit in 48 MiB of L2 together, number
// the units split-fastest with S near sqrt(slots), so that the units in
// flight share about slots / S row blocks and S W tiles.
#ifndef CKL_FWD_H_L2_MIB
#define CKL_FWD_H_L2_MIB 48
#endif
void forward_schedule(TcParams& p, int64_t d, int eb, int slots) {
  const int64_t hblk = kMB * d * eb;
  if (static_cast<int64_t>(p.n_rb) * hblk > (int64_t(CKL_FWD_H_L2_MIB) << 20)) {
    p.split_fast = 1;
    p.S = choose_splits(p.n_rb, p.n_vt, slots, 4, 16);
  } else {
    p.split_fast = 0;
    p.S = choose_splits(p.n_rb, p.n_vt, slots);
  }
  p.n_units = p.n_rb * p.S;
}

int pick_bn(int64_t d) {
  int best = 256;
  double best_cost = static_cast<double>(cdiv(d, 256) * 256);
  for (int bn : {192, 128, 64}) {
    if (kPair && bn % 128 != 0) continue;  // each CTA of a pair stages bn/2 columns
    const double slow = bn >= 192 ? 1.0 : bn == 128 ? 1.5 : 2.0;
    const double cost = static_cast<double>(cdiv(d, bn) * bn) * slow;
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

int status_from_word(int32_t w) {
  if (w & CKL_DEV_BAD_INDEX) return CKL_ERR_BAD_INDEX;
  if (w & CKL_DEV_BAD_LOGP) return CKL_ERR_BAD_LOGP;
  if (w & CKL_DEV_TIMEOUT) return CKL_ERR_TIMEOUT;
  return CKL_OK;
}

// Header reset, then S1 (prep) into the workspace at w8 laid out by L.
int clear_and_prep(const int32_t* idx, const float* logp, const uint8_t* mask, int64_t T,
                   int32_t K, int64_t V, uint8_t* w8, const Layout& L, cudaStream_t st,
                   ckl_trace* trace) {
  if (cudaMemsetAsync(w8, 0, kHeaderBytes, st) != cudaSuccess) return CKL_ERR_CUDA;
  if (T > 0) {
    Header* hdr = reinterpret_cast<Header*>(w8);
    TraceScope ts(trace, st, CKL_KERNEL_PREP);
    if (K <= ckl::PREP_MAXK) {
      const unsigned grid = static_cast<unsigned>(cdiv(T, ckl::PREP_WARPS));
      ckl::prep_kernel<<<grid, ckl::PREP_WARPS * 32, 0, st>>>(
          idx, logp, mask, T, K, V, reinterpret_cast<int2*>(w8 + L.pairs),
          reinterpret_cast<float*>(w8 + L.hp), &hdr->status, &hdr->countN);
    } else {
      ckl::prep_large_kernel<<<static_cast<unsigned>(T), ckl::PREPL_THREADS, 0, st>>>(
          idx, logp, mask, T, K, V, reinterpret_cast<int2*>(w8 + L.pairs),
          reinterpret_cast<float*>(w8 + L.hp), &hdr->status, &hdr->countN);
    }
    if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
  }
  return CKL_OK;
}

// Shared front half of forward and backward: checks, header reset, prep.
int common_prep(const void* H, const void* W, const int32_t* idx, const float* logp,
                const uint8_t* mask, int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk,
                void* ws, size_t ws_bytes, cudaStream_t st, ckl_trace* trace, DevInfo& di,
                Layout& L, bool single_pass = false, int eb = 2, int64_t v_valid = -1) {
  if (!sizes_ok(T, d, V, K, chunk)) return CKL_ERR_INVALID_ARG;
  // H, topk_idx and topk_logp may be NULL only for an empty batch.
  if (!W || !ws || (T > 0 && (!H || !idx || !logp))) return CKL_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(W) || !aligned16(ws) || !aligned4(idx) || !aligned4(logp))
    return CKL_ERR_INVALID_ARG;
  if (K > ckl::PREP_MAXK_LARGE) return CKL_ERR_UNSUPPORTED;
  L = layout(T, d, V, K, chunk, single_pass, eb);
  if (ws_bytes < L.total) return CKL_ERR_WORKSPACE;
  if (!device_info(di)) return CKL_ERR_CUDA;
  if (di.major != 10) return CKL_ERR_UNSUPPORTED;
  if (!encode_fn()) return CKL_ERR_CUDA;
  return clear_and_prep(idx, logp, mask, T, K, v_valid < 0 ? V : v_valid,
                        static_cast<uint8_t*>(ws), L, st, trace);
}

void fill_common(TcParams& p, uint8_t* w8, const Layout& L, int64_t T, int64_t d, int64_t V,
                 int32_t K, const uint8_t* mask) {
  Header* hdr = reinterpret_cast<Header*>(w8);
  p.T = static_cast<int32_t>(T);
  p.d = static_cast<int32_t>(d);
  p.V = static_cast<int32_t>(V);
  p.K = K;
  p.n_vt = static_cast<int32_t>(cdiv(V, ckl::BN_V));
  p.pairs = reinterpret_cast<const int2*>(w8 + L.pairs);
  p.partials = reinterpret_cast<float4*>(w8 + L.partials);
  p.mask = mask;
  p.status = &hdr->status;
  p.countN = &hdr->countN;
}

// H_c^T for rows [r0, r0 + rows): the K-major B operand of the dW GEMM.
template <bool F32>
int transpose_rows(const void* H, int64_t d, int64_t r0, int64_t rows, uint8_t* w8,
                   const Layout& L, cudaStream_t st, ckl_trace* trace) {
  using E = std::conditional_t<F32, float, uint16_t>;
  TraceScope ts(trace, st, CKL_KERNEL_OTHER);
  const dim3 grid(static_cast<unsigned>(cdiv(d, 32)), static_cast<unsigned>(cdiv(rows, 32)));
  ckl::transpose_rows_kernel<E><<<grid, 256, 0, st>>>(
      static_cast<const E*>(H) + r0 * d, static_cast<int>(rows), static_cast<int>(d),
      reinterpret_cast<E*>(w8 + L.hct), static_cast<int>(L.pitch_t));
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

// dZ of one block: rows [r0, r0 + rows) x vocabulary columns [v_lo, v_lo + cols)
// (v_lo a multiple of 256), recomputed from H and W, into panels
// [ceil(cols/PW)][prow][PW] at the start of the dZ buffer (PW = 64 bf16 or
// 32 fp32 columns: 128 bytes).
template <bool F32>
int dz_block(const void* H, const void* W, const uint8_t* mask, const float* lse, int64_t T,
             int64_t d, int64_t V, int32_t K, int64_t r0, int64_t rows, int64_t prow,
             int64_t v_lo, int64_t cols, uint8_t* w8, const Layout& L, const DevInfo& di,
             cudaStream_t st, ckl_trace* trace, int64_t v_off = 0) {
  constexpr int eb = F32 ? 4 : 2;
  constexpr uint32_t PW = kKE<F32>;
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, w8, L, T, d, V, K, mask);
  p.rows = static_cast<int32_t>(rows);
  p.row0 = static_cast<int32_t>(r0);
  p.n_rb = static_cast<int32_t>(cdiv(rows, kMB));
  p.vt0 = static_cast<int32_t>(v_lo / ckl::BN_V);
  p.n_vt = static_cast<int32_t>(cdiv(cols, ckl::BN_V));
  p.S = 1;
  p.n_units = p.n_rb * p.n_vt;  // tiles, dealt out round-robin
  p.lse = lse;
  p.v_off = static_cast<int32_t>(v_off);
  const uint8_t* Hr = static_cast<const uint8_t*>(H) + r0 * d * eb;
  if (!map2d(&p.tm[0], kDT<F32>, Hr, d, rows, d * eb, kKE<F32>, ckl::BM,
             CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map2d(&p.tm[1], kDT<F32>, W, d, V, d * eb, kKE<F32>, ckl::BN_V / kSlotCTAs,
             CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map3d(&p.tm[2], kDT<F32>, w8 + L.dz, PW, rows, cdiv(cols, PW), 128, prow * 128, 32,
             ckl::BM, F32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return CKL_ERR_CUDA;
  TraceScope ts(trace, st, CKL_KERNEL_BWD_DZ);
  return launch_tc<ckl::MODE_DZ, F32>(p, p.n_units, di, st);
}

// Quotas of dW tiles for the round-dealt schedule (dw_mode 1): slots below
// r5 = n5 mod G hold one more dH unit (c5 k-blocks later to start).  Water-
// filling: the smallest finishing k-block t whose per-class quotas
// floor((t - start) / (c6 + 1)) cover n6 tiles, then the excess trimmed from
// the class that finishes later.  Class quota Q for its first E slots and
// Q - 1 for the rest.
void dw_round_quotas(TcParams& p, int64_t G) {
  const int64_t c = p.c6 + 1;
  const int64_t a5 = p.n5 / G, r5 = p.n5 % G;
  const int64_t s_l = a5 * p.c5, s_h = s_l + p.c5;
  const int64_t nl = G - r5, nh = r5;
  auto tot = [&](int64_t t, int64_t& ql, int64_t& qh) {
    ql = t > s_l ? (t - s_l) / c : 0;
    qh = t > s_h ? (t - s_h) / c : 0;
    return nl * ql + nh * qh;
  };
  int64_t lo = 0, hi = s_h + (static_cast<int64_t>(p.n6) + 1) * c, ql = 0, qh = 0;
  while (lo < hi) {
    const int64_t mid = (lo + hi) / 2;
    if (tot(mid, ql, qh) >= p.n6) hi = mid;
    else lo = mid + 1;
  }
  int64_t ex = tot(lo, ql, qh) - p.n6;
  int64_t El = nl, Eh = nh;
  while (ex > 0) {
    const int64_t end_l = (ql > 0 && El > 0) ? s_l + ql * c : -1;
    const int64_t end_h = (qh > 0 && Eh > 0) ? s_h + qh * c : -1;
    if (end_l >= end_h) {
      const int64_t take = std::min(ex, El);
      El -= take;
      ex -= take;
      if (El == 0 && ql > 0) { --ql; El = nl; }
    } else {
      const int64_t take = std::min(ex, Eh);
      Eh -= take;
      ex -= take;
      if (Eh == 0 && qh > 0) { --qh; Eh = nh; }
    }
  }
  p.dw_Ql = static_cast<int32_t>(ql);
  p.dw_El = static_cast<int32_t>(El);
  p.dw_Qh = static_cast<int32_t>(qh);
  p.dw_Eh = static_cast<int32_t>(Eh);
}

// dH and dW of one block from its dZ panels (and H_c^T of its rows), one
// merged GEMM launch.  dh_mode 0 writes dH rows as bf16 (dh_out = dH + r0 d);
// 1 stores and 2 adds the block's fp32 share into dh_out (the partial dH of
// a sliced row chunk, or the fp32 entry points' dH rows).  dw_store 1 stores
// the block's dW rows, 0 adds.
template <bool F32>
int dhdw_block(const void* W, const uint8_t* mask, int64_t T, int64_t d, int64_t V, int32_t K,
               int64_t r0, int64_t rows, int64_t prow, int64_t v_lo, int64_t cols, int dh_mode,
               int dw_store, const float* grad_loss, void* dh_out, float* dW, uint8_t* w8,
               const Layout& L, const DevInfo& di, cudaStream_t st, ckl_trace* trace) {
  constexpr int eb = F32 ? 4 : 2;
  constexpr uint32_t KE = kKE<F32>;  // also the panel width
  void* dz = w8 + L.dz;
  const int bn = pick_bn(d);
  const int64_t npan = cdiv(cols, KE);
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, w8, L, T, d, V, K, mask);
  p.rows = static_cast<int32_t>(rows);
  p.row0 = static_cast<int32_t>(r0);
  p.bn = bn;
  p.n_nt = static_cast<int32_t>(cdiv(d, bn));
  p.n_mt = static_cast<int32_t>(cdiv(cols, kMB));
  p.n5 = static_cast<int32_t>(cdiv(rows, kMB)) * p.n_nt;
  p.n6 = p.n_mt * p.n_nt;
  p.c5 = static_cast<int32_t>(npan);
  p.c6 = static_cast<int32_t>(cdiv(rows, KE));
  p.dw_store = dw_store;
  p.v_lo = static_cast<int32_t>(v_lo);
  p.dh_mode = dh_mode;
  p.grad_loss = grad_loss;
  // dW tiles: contiguous per slot while every slot's dZ panels (kMB x rows
  // per vocabulary block) fit in L2 together, else dealt in rounds
  const int64_t G = std::min<int64_t>(di.slots[ckl::MODE_DHDW], p.n5 + p.n6);
  p.dw_mode = (kMB * rows * eb * G > (int64_t(48) << 20)) ? 1 : 0;
  if (p.dw_mode == 1) dw_round_quotas(p, G);
  const bool dh_low = (dh_mode == 0);  // bf16 dH
  // the MN-major operands (W for dH, dZ^T for dW): tf32 ones take the 128-byte
  // swizzle with 32-byte chunks, the only MN-major layout of kind::tf32
  constexpr CUtensorMapSwizzle mn_sw =
      F32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  // W as the dH GEMM's MN-major B operand: viewed as [d / KE][V][KE] when d
  // is a multiple of KE, so that one box carries a CTA's half_n columns per
  // stage (half_n / KE atoms, ATOM_B apart); otherwise one 2-D box per atom
  p.w3d = (d % KE == 0 &&
           map3d2(&p.tm[1], kDT<F32>, W, KE, V, d / KE, d * eb, KE * eb, KE, KE,
                  static_cast<uint32_t>(bn / kSlotCTAs / KE), mn_sw))
              ? 1 : 0;
  if (!p.w3d && !map2d(&p.tm[1], kDT<F32>, W, d, V, d * eb, KE, KE, mn_sw)) return CKL_ERR_CUDA;
  if (!map3d(&p.tm[0], kDT<F32>, dz, KE, rows, npan, 128, prow * 128, KE, ckl::BM,
             CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map3d2(&p.tm[2], kDT<F32>, dz, KE, rows, npan, 128, prow * 128, KE, KE,
              static_cast<uint32_t>(ckl::BM / KE), mn_sw) ||
      !map2d(&p.tm[3], kDT<F32>, w8 + L.hct, rows, d, L.pitch_t * eb, KE, bn / kSlotCTAs,
             CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map2d(&p.tm[4], dh_low ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
             dh_out, d, rows, d * (dh_low ? 2 : 4), 32, ckl::BM,
             dh_low ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map2d(&p.tm[5], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dW, d, V, d * 4, 32, ckl::BM,
             CU_TENSOR_MAP_SWIZZLE_128B))
    return CKL_ERR_CUDA;
  TraceScope ts(trace, st, CKL_KERNEL_BWD_DHDW);
  return launch_tc<ckl::MODE_DHDW, F32>(p, p.n5 + p.n6, di, st);
}

// S2-S4 once the prep has run: the logit GEMM with its online log-sum-exp and
// teacher gather, then the combine (lse, loss).  T = 0 only writes loss = 0.
template <bool F32>
int forward_gemm_combine(const void* H, const void* W, const uint8_t* mask, int64_t T, int64_t d,
                         int64_t V, int32_t K, float* loss, float* lse, uint8_t* w8,
                         const Layout& L, const DevInfo& di, cudaStream_t st, ckl_trace* trace) {
  constexpr int eb = F32 ? 4 : 2;
  Header* hdr = reinterpret_cast<Header*>(w8);
  if (T == 0) {
    TraceScope ts(trace, st, CKL_KERNEL_OTHER);
    ckl::zero_loss_kernel<<<1, 1, 0, st>>>(loss);
    return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
  }
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, w8, L, T, d, V, K, mask);
  p.rows = static_cast<int32_t>(T);
  p.row0 = 0;
  p.n_rb = static_cast<int32_t>(cdiv(T, kMB));
  forward_schedule(p, d, eb, di.slots[ckl::MODE_FWD]);
  if (!map2d(&p.tm[0], kDT<F32>, H, d, T, d * eb, kKE<F32>, ckl::BM,
             CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map2d(&p.tm[1], kDT<F32>, W, d, V, d * eb, kKE<F32>, ckl::BN_V / kSlotCTAs,
             CU_TENSOR_MAP_SWIZZLE_128B))
    return CKL_ERR_CUDA;
  {
    TraceScope ts(trace, st, CKL_KERNEL_FWD_GEMM);
    if (launch_tc<ckl::MODE_FWD, F32>(p, p.n_units, di, st) != CKL_OK) return CKL_ERR_CUDA;
  }
  {
    TraceScope ts(trace, st, CKL_KERNEL_FWD_COMBINE);
    const unsigned grid = static_cast<unsigned>(cdiv(T, ckl::COMBINE_THREADS));
    ckl::combine_kernel<<<grid, ckl::COMBINE_THREADS, 0, st>>>(
        reinterpret_cast<const float4*>(w8 + L.partials), p.S, p.S, 1,
        reinterpret_cast<const float*>(w8 + L.hp), mask, T, lse,
        reinterpret_cast<double*>(w8 + L.blocksums), &hdr->ticket, &hdr->countN, loss,
        &hdr->numer);
    if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
  }
  return CKL_OK;
}

// The forward (S1-S4) on bf16 or fp32 H and W.
template <bool F32>
int forward_impl(const void* H, const void* W, const int32_t* topk_idx, const float* topk_logp,
                 const uint8_t* mask, int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk,
                 float* loss, float* lse, void* workspace, size_t workspace_bytes, void* stream,
                 ckl_trace* trace) {
  if (!loss || !aligned4(loss) || (T > 0 && (!lse || !aligned4(lse)))) return CKL_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevInfo di;
  Layout L;
  int rc = common_prep(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, workspace,
                       workspace_bytes, st, trace, di, L, false, F32 ? 4 : 2);
  if (rc != CKL_OK) return rc;
  return forward_gemm_combine<F32>(H, W, mask, T, d, V, K, loss, lse,
                                  static_cast<uint8_t*>(workspace), L, di, st, trace);
}

// The blocked backward (S0, S1, S5-S7) on bf16 or fp32 H and W; dH is bf16
// or fp32 like H.  For a vocabulary shard (W = rows [v_off, v_off + V) of a
// head of v_valid rows), dH_f32 = true: dH is this shard's fp32 share, summed
// over the shards by the caller.
template <bool F32>
int backward_impl(const void* H, const void* W, const int32_t* topk_idx, const float* topk_logp,
                  const uint8_t* mask, int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk,
                  const float* lse, const float* grad_loss, void* dH, float* dW,
                  int32_t accumulate_dW, void* workspace, size_t workspace_bytes, void* stream,
                  ckl_trace* trace, ckl_dw_ready_fn on_dw_ready, void* user,
                  int64_t v_valid = -1, int64_t v_off = 0, bool dh_f32 = F32) {
  constexpr int eb = F32 ? 4 : 2;
  if (!dW || !aligned16(dW)) return CKL_ERR_INVALID_ARG;
  if (T > 0 && (!lse || !aligned4(lse) || !dH || !aligned16(dH))) return CKL_ERR_INVALID_ARG;
  if (grad_loss && !aligned4(grad_loss)) return CKL_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevInfo di;
  Layout L;
  int rc = common_prep(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, workspace,
                       workspace_bytes, st, trace, di, L, false, eb, v_valid);
  if (rc != CKL_OK) return rc;
  if (T == 0) {
    if (!accumulate_dW &&
        cudaMemsetAsync(dW, 0, static_cast<size_t>(V) * d * sizeof(float), st) != cudaSuccess)
      return CKL_ERR_CUDA;
    if (on_dw_ready) on_dw_ready(0, V, user);
    return CKL_OK;
  }
  uint8_t* w8 = static_cast<uint8_t*>(workspace);
  const Plan P = plan_backward(T, d, V, L);
  float* dh32 = reinterpret_cast<float*>(w8 + L.dh32);
  for (int64_t r0 = 0; r0 < T; r0 += P.Cr) {
    const int64_t rows = std::min(P.Cr, T - r0);
    rc = transpose_rows<F32>(H, d, r0, rows, w8, L, st, trace);
    if (rc != CKL_OK) return rc;
    const int dw_store = (r0 == 0 && !accumulate_dW) ? 1 : 0;
    for (int64_t s = 0; s < P.n; ++s) {
      const int64_t v_lo = s * P.Sv;
      const int64_t cols = std::min(P.Sv, V - v_lo);
      rc = dz_block<F32>(H, W, mask, lse, T, d, V, K, r0, rows, P.Cr, v_lo, cols, w8, L, di,
                         st, trace, v_off);
      if (rc != CKL_OK) return rc;
      // bf16 dH: one slab writes it, several sum into the fp32 partial first;
      // fp32 dH: the slabs store / add into the output itself
      int dh_mode;
      void* dh_out;
      if (dh_f32) {
        dh_mode = (s == 0) ? 1 : 2;
        dh_out = static_cast<uint8_t*>(dH) + r0 * d * 4;
      } else {
        dh_mode = (P.n == 1) ? 0 : (s == 0 ? 1 : 2);
        dh_out = (P.n == 1) ? static_cast<void*>(static_cast<uint8_t*>(dH) + r0 * d * 2)
                            : static_cast<void*>(dh32);
      }
      rc = dhdw_block<F32>(W, mask, T, d, V, K, r0, rows, P.Cr, v_lo, cols, dh_mode, dw_store,
                           grad_loss, dh_out, dW, w8, L, di, st, trace);
      if (rc != CKL_OK) return rc;
      // the last row chunk's launch is the last to write these dW rows
      if (on_dw_ready && r0 + rows == T) on_dw_ready(v_lo, v_lo + cols, user);
    }
    if (!dh_f32 && P.n > 1) {
      // dH rows of this chunk: the fp32 sum over its slabs, rounded once
      TraceScope ts(trace, st, CKL_KERNEL_OTHER);
      const int64_t n4 = rows * d / 4;
      const unsigned grid = static_cast<unsigned>(std::min<int64_t>(cdiv(n4, 256), 4 * di.sms));
      ckl::dh_convert_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(dh32), n4,
                                                   reinterpret_cast<uint2*>(
                                                       static_cast<uint8_t*>(dH) + r0 * d * 2));
      if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
    }
  }
  return CKL_OK;
}

}  // namespace

extern "C" {

size_t ckl_workspace_bytes(int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk) {
  if (!sizes_ok(T, d, V, K, chunk)) return 0;
  return layout(T, d, V, K, chunk, false).total;
}

int ckl_forward(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                int32_t K, int64_t chunk, float* loss, float* lse, void* workspace,
                size_t workspace_bytes, void* stream, ckl_trace* trace) {
  return forward_impl<false>(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, loss, lse,
                             workspace, workspace_bytes, stream, trace);
}

int ckl_backward(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                 const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                 int32_t K, int64_t chunk, const float* lse, const float* grad_loss,
                 uint16_t* dH, float* dW, int32_t accumulate_dW, void* workspace,
                 size_t workspace_bytes, void* stream, ckl_trace* trace) {
  return ckl_backward_ex(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, lse, grad_loss, dH,
                         dW, accumulate_dW, workspace, workspace_bytes, stream, trace, nullptr,
                         nullptr);
}

int ckl_backward_ex(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                    const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                    int32_t K, int64_t chunk, const float* lse, const float* grad_loss,
                    uint16_t* dH, float* dW, int32_t accumulate_dW, void* workspace,
                    size_t workspace_bytes, void* stream, ckl_trace* trace,
                    ckl_dw_ready_fn on_dw_ready, void* user) {
  return backward_impl<false>(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, lse, grad_loss,
                              dH, dW, accumulate_dW, workspace, workspace_bytes, stream, trace,
                              on_dw_ready, user);
}

size_t ckl_workspace_bytes_f32(int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk) {
  if (!sizes_ok(T, d, V, K, chunk)) return 0;
  return layout(T, d, V, K, chunk, false, 4).total;
}

int ckl_forward_f32(const float* H, const float* W, const int32_t* topk_idx,
                    const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                    int32_t K, int64_t chunk, float* loss, float* lse, void* workspace,
                    size_t workspace_bytes, void* stream, ckl_trace* trace) {
  return forward_impl<true>(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, loss, lse,
                            workspace, workspace_bytes, stream, trace);
}

int ckl_backward_f32(const float* H, const float* W, const int32_t* topk_idx,
                     const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d,
                     int64_t V, int32_t K, int64_t chunk, const float* lse,
                     const float* grad_loss, float* dH, float* dW, int32_t accumulate_dW,
                     void* workspace, size_t workspace_bytes, void* stream, ckl_trace* trace) {
  return backward_impl<true>(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, lse, grad_loss,
                             dH, dW, accumulate_dW, workspace, workspace_bytes, stream, trace,
                             nullptr, nullptr);
}

int ckl_backward_plan(int64_t T, int64_t d, int64_t V, int32_t K, int64_t chunk,
                      int64_t* plan) {
  if (!plan || !sizes_ok(T, d, V, K, chunk)) return CKL_ERR_INVALID_ARG;
  const Layout L = layout(T, d, V, K, chunk, false);
  const Plan P = plan_backward(T, d, V, L);
  plan[0] = P.Cr;
  plan[1] = P.Sv;
  plan[2] = P.n;
  return CKL_OK;
}

size_t ckl_single_pass_workspace_bytes(int64_t T, int64_t d, int64_t V, int32_t K,
                                       int64_t chunk) {
  if (!sizes_ok(T, d, V, K, chunk)) return 0;
  return layout(T, d, V, K, chunk, true).total;
}

int ckl_forward_backward(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                         const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d,
                         int64_t V, int32_t K, int64_t chunk, const float* grad_loss, float* loss,
                         float* lse, uint16_t* dH, float* dW, int32_t accumulate_dW,
                         void* workspace, size_t workspace_bytes, void* stream,
                         ckl_trace* trace) {
  if (!loss || !aligned4(loss) || !dW || !aligned16(dW)) return CKL_ERR_INVALID_ARG;
  if (T > 0 && (!lse || !aligned4(lse) || !dH || !aligned16(dH))) return CKL_ERR_INVALID_ARG;
  if (grad_loss && !aligned4(grad_loss)) return CKL_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevInfo di;
  Layout L;
  int rc = common_prep(H, W, topk_idx, topk_logp, mask, T, d, V, K, chunk, workspace,
                       workspace_bytes, st, trace, di, L, true);
  if (rc != CKL_OK) return rc;
  if (T == 0) {
    if (!accumulate_dW &&
        cudaMemsetAsync(dW, 0, static_cast<size_t>(V) * d * sizeof(float), st) != cudaSuccess)
      return CKL_ERR_CUDA;
    TraceScope ts(trace, st, CKL_KERNEL_OTHER);
    ckl::zero_loss_kernel<<<1, 1, 0, st>>>(loss);
    return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
  }
  uint8_t* w8 = static_cast<uint8_t*>(workspace);
  Header* hdr = reinterpret_cast<Header*>(w8);
  float* z = reinterpret_cast<float*>(w8 + L.z);
  float* rowloss = reinterpret_cast<float*>(w8 + L.rowloss);
  const int64_t grp = L.sp_rows;  // rows of one dH / dW launch: kSpGroup chunks
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    const int64_t rows = std::min<int64_t>(chunk, T - c0);
    const int64_t g0 = c0 / grp * grp;  // first row of this chunk's group
    const uint16_t* Hc = H + c0 * d;
    // ---- logits of this chunk, once: online log-sum-exp + gather partials and fp32 z
    TcParams p;
    std::memset(&p, 0, sizeof(p));
    fill_common(p, w8, L, T, d, V, K, mask);
    p.rows = static_cast<int32_t>(rows);
    p.row0 = static_cast<int32_t>(c0);
    p.n_rb = static_cast<int32_t>(cdiv(rows, kMB));
    forward_schedule(p, d, 2, di.slots[ckl::MODE_FWDZ]);
    if (!map2d(&p.tm[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Hc, d, rows, d * 2, ckl::BK, ckl::BM,
               CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map2d(&p.tm[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, d, V, d * 2, ckl::BK,
               ckl::BN_V / kSlotCTAs, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map2d(&p.tm[2], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, z, V, rows, L.zpitch * 4, 32, ckl::BM,
               CU_TENSOR_MAP_SWIZZLE_128B))
      return CKL_ERR_CUDA;
    {
      TraceScope ts(trace, st, CKL_KERNEL_SP_GEMM);
      if (launch_tc<ckl::MODE_FWDZ>(p, p.n_units, di, st) != CKL_OK) return CKL_ERR_CUDA;
    }
    // ---- lse, the rows' loss terms and dZ from the stored logits
    {
      TraceScope ts(trace, st, CKL_KERNEL_SP_ROWS);
      ckl::zrow_kernel<<<static_cast<unsigned>(rows), ckl::ZROW_THREADS, 0, st>>>(
          z, L.zpitch, reinterpret_cast<const float4*>(w8 + L.partials), p.S,
          reinterpret_cast<const float*>(w8 + L.hp), mask,
          reinterpret_cast<const int2*>(w8 + L.pairs), K, static_cast<int>(V), c0, grp, c0 - g0,
          lse, rowloss, reinterpret_cast<uint16_t*>(w8 + L.dz));
      if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
    }
    // ---- dH and dW once the group's dZ is complete
    if (c0 + rows == T || c0 + rows == g0 + grp) {
      const int64_t grows = c0 + rows - g0;
      rc = transpose_rows<false>(H, d, g0, grows, w8, L, st, trace);
      if (rc != CKL_OK) return rc;
      rc = dhdw_block<false>(W, mask, T, d, V, K, g0, grows, grp, 0, V, 0,
                             (g0 == 0 && !accumulate_dW) ? 1 : 0, grad_loss, dH + g0 * d, dW,
                             w8, L, di, st, trace);
      if (rc != CKL_OK) return rc;
    }
  }
  {
    TraceScope ts(trace, st, CKL_KERNEL_FWD_COMBINE);
    ckl::rowsum_loss_kernel<<<1, ckl::ROWSUM_THREADS, 0, st>>>(rowloss, T, &hdr->countN, loss,
                                                                &hdr->numer);
    if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
  }
  return CKL_OK;
}

int ckl_topk_cache(const uint16_t* teacher_logits, int64_t T, int64_t V, int32_t K,
                   int32_t* topk_idx, float* topk_logp, int32_t* device_status, void* stream) {
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (T < 0 || T >= lim || V < 1 || V >= lim || K < 1 || K > V) return CKL_ERR_INVALID_ARG;
  if (K > ckl::TK_CAP) return CKL_ERR_UNSUPPORTED;
  if (T > 0 && (!teacher_logits || !topk_idx || !topk_logp)) return CKL_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(teacher_logits) & 1u) || !aligned4(topk_idx) ||
      !aligned4(topk_logp) || !aligned4(device_status))
    return CKL_ERR_INVALID_ARG;
  if (T * V >= (int64_t(1) << 62) / 2) return CKL_ERR_INVALID_ARG;
  DevInfo di;
  if (!device_info(di)) return CKL_ERR_CUDA;
  if (di.major != 10) return CKL_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (device_status && cudaMemsetAsync(device_status, 0, sizeof(int32_t), st) != cudaSuccess)
    return CKL_ERR_CUDA;
  if (T == 0) return CKL_OK;
  const int vec8 = (V % 8 == 0 && aligned16(teacher_logits)) ? 1 : 0;
  const int grid = static_cast<int>(std::min<int64_t>(T, static_cast<int64_t>(di.sms) * 2));
  if (K <= ckl::TS_THREADS) {
    // the vector maxima in dynamic shared memory (2 bytes per 8 logits, in
    // whole passes of the block) when they fit
    const int mark = (vec8 && V <= ckl::TS_MARK_MAX_V) ? 1 : 0;
    const int64_t passes = (V / 8 + ckl::TS_PER_PASS - 1) / ckl::TS_PER_PASS;
    const size_t dyn = mark ? static_cast<size_t>(passes) * ckl::TS_THREADS * 8 : 0;
    if (cudaFuncSetAttribute(ckl::topk_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ckl::TS_MARK_MAX_V / 8 * 2) != cudaSuccess)
      return CKL_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ckl::topk_stream_kernel,
                                                      ckl::TS_THREADS, dyn) != cudaSuccess ||
        per_sm < 1)
      return CKL_ERR_CUDA;
    per_sm = std::min(per_sm, ckl::TS_BLOCKS);
    const int sgrid = static_cast<int>(std::min<int64_t>(T, static_cast<int64_t>(di.sms) * per_sm));
    ckl::topk_stream_kernel<<<sgrid, ckl::TS_THREADS, dyn, st>>>(
        teacher_logits, T, static_cast<int>(V), K, vec8, mark, topk_idx, topk_logp, device_status);
    if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
    ckl::topk_fallback_kernel<<<grid, ckl::TK_THREADS, 0, st>>>(
        teacher_logits, T, static_cast<int>(V), K, vec8, topk_idx, topk_logp, device_status);
  } else
    ckl::topk_cache_kernel<<<grid, ckl::TK_THREADS, 0, st>>>(
        teacher_logits, T, static_cast<int>(V), K, vec8, topk_idx, topk_logp, device_status);
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_find_duplicate_ids(const int32_t* topk_idx, int64_t T, int32_t K,
                           int32_t* first_dup_row, void* stream) {
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (T < 0 || T >= lim || K < 1) return CKL_ERR_INVALID_ARG;
  if (K > ckl::PREP_MAXK_LARGE) return CKL_ERR_UNSUPPORTED;
  if (!first_dup_row || !aligned4(first_dup_row) || (T > 0 && (!topk_idx || !aligned4(topk_idx))))
    return CKL_ERR_INVALID_ARG;
  if (T * static_cast<int64_t>(K) >= lim) return CKL_ERR_INVALID_ARG;
  DevInfo di;
  if (!device_info(di)) return CKL_ERR_CUDA;
  if (di.major != 10) return CKL_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(first_dup_row, 0xFF, sizeof(int32_t), st) != cudaSuccess)  // -1
    return CKL_ERR_CUDA;
  if (T == 0) return CKL_OK;
  const int grid = static_cast<int>(std::min<int64_t>(T, static_cast<int64_t>(di.sms) * 8));
  ckl::dup_ids_kernel<<<grid, ckl::DUP_THREADS, 0, st>>>(topk_idx, T, K,
                                                        reinterpret_cast<uint32_t*>(first_dup_row));
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_selftest_wait_timeout(int64_t limit_ns, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (!workspace || !aligned16(workspace) || workspace_bytes < kHeaderBytes)
    return CKL_ERR_INVALID_ARG;
  if (limit_ns < 1000000 || limit_ns > 4000000000ll) return CKL_ERR_INVALID_ARG;
  DevInfo di;
  if (!device_info(di)) return CKL_ERR_CUDA;
  if (di.major != 10) return CKL_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, st) != cudaSuccess) return CKL_ERR_CUDA;
  Header* hdr = static_cast<Header*>(workspace);
  ckl::wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(&hdr->status,
                                                      static_cast<uint64_t>(limit_ns));
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_forward_vocab_shard(const uint16_t* H, const uint16_t* W_shard, const int32_t* topk_idx,
                            const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d,
                            int64_t V, int64_t v_begin, int64_t v_end, int32_t K, int64_t chunk,
                            float* row_partials, void* workspace, size_t workspace_bytes,
                            void* stream, ckl_trace* trace) {
  if (v_begin < 0 || v_end <= v_begin || v_end > V || !sizes_ok(T, d, V, K, chunk))
    return CKL_ERR_INVALID_ARG;
  if (T > 0 && (!row_partials || !aligned16(row_partials))) return CKL_ERR_INVALID_ARG;
  const int64_t Vs = v_end - v_begin;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevInfo di;
  Layout L;
  int rc = common_prep(H, W_shard, topk_idx, topk_logp, mask, T, d, Vs, K, chunk, workspace,
                       workspace_bytes, st, trace, di, L, false, 2, V);
  if (rc != CKL_OK || T == 0) return rc;
  uint8_t* w8 = static_cast<uint8_t*>(workspace);
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, w8, L, T, d, Vs, K, mask);
  p.rows = static_cast<int32_t>(T);
  p.n_rb = static_cast<int32_t>(cdiv(T, kMB));
  p.v_off = static_cast<int32_t>(v_begin);
  forward_schedule(p, d, 2, di.slots[ckl::MODE_FWD]);
  if (!map2d(&p.tm[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, H, d, T, d * 2, ckl::BK, ckl::BM,
             CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map2d(&p.tm[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_shard, d, Vs, d * 2, ckl::BK,
             ckl::BN_V / kSlotCTAs, CU_TENSOR_MAP_SWIZZLE_128B))
    return CKL_ERR_CUDA;
  {
    TraceScope ts(trace, st, CKL_KERNEL_FWD_GEMM);
    if (launch_tc<ckl::MODE_FWD>(p, p.n_units, di, st) != CKL_OK) return CKL_ERR_CUDA;
  }
  TraceScope ts(trace, st, CKL_KERNEL_FWD_COMBINE);
  ckl::merge_splits_kernel<<<static_cast<unsigned>(cdiv(T, ckl::COMBINE_THREADS)),
                             ckl::COMBINE_THREADS, 0, st>>>(
      reinterpret_cast<const float4*>(w8 + L.partials), p.S, T,
      reinterpret_cast<float4*>(row_partials));
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_combine_vocab_shards(const float* gathered, int32_t g, const uint8_t* mask, int64_t T,
                             int32_t K, float* loss, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream, ckl_trace* trace) {
  if (g < 1 || T < 0 || K < 1 || !loss || !aligned4(loss) || !workspace ||
      !aligned16(workspace) || (T > 0 && (!gathered || !aligned16(gathered) || !lse ||
                                          !aligned4(lse))))
    return CKL_ERR_INVALID_ARG;
  const Layout L = forward_layout(T, K);
  if (workspace_bytes < L.total) return CKL_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(workspace);
  Header* hdr = reinterpret_cast<Header*>(w8);
  if (T == 0) {
    TraceScope ts(trace, st, CKL_KERNEL_OTHER);
    ckl::zero_loss_kernel<<<1, 1, 0, st>>>(loss);
    return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
  }
  if (cudaMemsetAsync(&hdr->ticket, 0, sizeof(hdr->ticket), st) != cudaSuccess)
    return CKL_ERR_CUDA;
  TraceScope ts(trace, st, CKL_KERNEL_FWD_COMBINE);
  ckl::combine_kernel<<<static_cast<unsigned>(cdiv(T, ckl::COMBINE_THREADS)),
                        ckl::COMBINE_THREADS, 0, st>>>(
      reinterpret_cast<const float4*>(gathered), g, 1, T,
      reinterpret_cast<const float*>(w8 + L.hp), mask, T, lse,
      reinterpret_cast<double*>(w8 + L.blocksums), &hdr->ticket, &hdr->countN, loss,
      &hdr->numer);
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_backward_vocab_shard(const uint16_t* H, const uint16_t* W_shard,
                             const int32_t* topk_idx, const float* topk_logp,
                             const uint8_t* mask, int64_t T, int64_t d, int64_t V,
                             int64_t v_begin, int64_t v_end, int32_t K, int64_t chunk,
                             const float* lse, const float* grad_loss, float* dH_partial,
                             float* dW_shard, int32_t accumulate_dW, void* workspace,
                             size_t workspace_bytes, void* stream, ckl_trace* trace) {
  if (v_begin < 0 || v_end <= v_begin || v_end > V || !sizes_ok(T, d, V, K, chunk))
    return CKL_ERR_INVALID_ARG;
  return backward_impl<false>(H, W_shard, topk_idx, topk_logp, mask, T, d, v_end - v_begin, K,
                              chunk, lse, grad_loss, dH_partial, dW_shard, accumulate_dW,
                              workspace, workspace_bytes, stream, trace, nullptr, nullptr, V,
                              v_begin, true);
}

int ckl_dh_to_bf16(const float* src, uint16_t* dst, int64_t n, void* stream) {
  if (n < 0 || n % 4 != 0 || (n > 0 && (!src || !dst || !aligned16(src) ||
                                        (reinterpret_cast<uintptr_t>(dst) & 7u))))
    return CKL_ERR_INVALID_ARG;
  if (n == 0) return CKL_OK;
  DevInfo di;
  if (!device_info(di)) return CKL_ERR_CUDA;
  const int64_t n4 = n / 4;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(cdiv(n4, 256), 4 * di.sms));
  ckl::dh_convert_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4*>(src), n4, reinterpret_cast<uint2*>(dst));
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_dp_local_stats(const void* workspace, double* stats, void* stream) {
  if (!workspace || !stats || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(stats) & 7u))
    return CKL_ERR_INVALID_ARG;
  const Header* hdr = static_cast<const Header*>(workspace);
  ckl::dp_local_stats_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(&hdr->numer,
                                                                          &hdr->countN, stats);
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_dp_finish(const double* stats, const float* grad_loss, float* loss, float* grad_local,
                  void* stream) {
  if (!stats || !loss || !grad_local || (reinterpret_cast<uintptr_t>(stats) & 7u) ||
      !aligned4(loss) || !aligned4(grad_local) || !aligned4(grad_loss))
    return CKL_ERR_INVALID_ARG;
  ckl::dp_finish_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(stats, grad_loss, loss,
                                                                      grad_local);
  return cudaGetLastError() == cudaSuccess ? CKL_OK : CKL_ERR_CUDA;
}

int ckl_read_device_status(const void* workspace, void* stream, int32_t* device_status) {
  if (!workspace || !device_status) return CKL_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t w = 0;
  if (cudaMemcpyAsync(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return CKL_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return CKL_ERR_CUDA;
  *device_status = w;
  return status_from_word(w);
}

const char* ckl_status_string(int32_t status) {
  switch (status) {
    case CKL_OK: return "ok";
    case CKL_ERR_INVALID_ARG: return "invalid argument (null pointer, size or alignment)";
    case CKL_ERR_UNSUPPORTED: return "unsupported (needs an sm_100 device and K <= 2048)";
    case CKL_ERR_WORKSPACE: return "workspace too small";
    case CKL_ERR_CUDA: return "CUDA call or kernel launch failed";
    case CKL_ERR_BAD_INDEX: return "teacher token id outside [0, V)";
    case CKL_ERR_BAD_LOGP: return "teacher log-prob NaN/+inf, or a row with none finite";
    case CKL_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out of time";
    case CKL_ERR_TOPK_TIES: return "too many teacher logits tie at a row's K-th value";
    case CKL_ERR_DUP_INDEX: return "a teacher token id repeated within a row";
    default: return "unknown status";
  }
}

int32_t ckl_version(void) { return kVersion; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward with library-owned static scratch, for callers that cannot
// allocate device memory.  The buffer is a file-scope device array; host code
// must never hand its name to a kernel (on the host the name is only a
// stand-in), so the real device address is looked up with
// cudaGetSymbolAddress on each device and kept.
namespace {

static __device__ __align__(256) uint8_t g_static_scratch[CKL_STATIC_SCRATCH_BYTES];

__global__ void copy_status_kernel(const int32_t* src, int32_t* dst) { *dst = *src; }

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_static_scratch on the current device, or null.  The
// address is kept per device together with the context it was looked up in;
// when the current context differs (after cudaDeviceReset, say, the module
// is loaded again) it is looked up again.
void* static_scratch_ptr() {
  static std::mutex mu;
  struct Entry {
    CUcontext ctx;
    void* ptr;
  };
  static Entry cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  Entry& e = cache[dev];
  CUcontext ctx = nullptr;
  CtxGetCurrentFn get = ctx_current_fn();
  const bool known = get && get(&ctx) == CUDA_SUCCESS && ctx != nullptr;
  if (e.ptr == nullptr || !known || ctx != e.ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    // the lookup makes the device's primary context current if none was
    if (get && get(&ctx) == CUDA_SUCCESS) e.ctx = ctx;
    e.ptr = p;
  }
  return e.ptr;
}

}  // namespace

extern "C" {

int ckl_forward_static_scratch(const uint16_t* H, const uint16_t* W, const int32_t* topk_idx,
                               const float* topk_logp, const uint8_t* mask, int64_t T, int64_t d,
                               int64_t V, int32_t K, float* loss, float* lse,
                               int32_t* device_status, void* stream) {
  if (!sizes_ok(T, d, V, K, 1)) return CKL_ERR_INVALID_ARG;
  if (!W || !loss || !aligned4(loss) || (T > 0 && (!H || !topk_idx || !topk_logp || !lse)))
    return CKL_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(W) || !aligned4(topk_idx) || !aligned4(topk_logp) ||
      !aligned4(lse) || !aligned4(device_status))
    return CKL_ERR_INVALID_ARG;
  if (K > ckl::PREP_MAXK_LARGE) return CKL_ERR_UNSUPPORTED;
  // The forward's own layout (as in ckl_forward, partials sized for the largest
  // split count), so the limit depends on T and K only; checked before any
  // device call.
  const Layout L = forward_layout(T, K);
  if (L.total > CKL_STATIC_SCRATCH_BYTES) return CKL_ERR_WORKSPACE;
  DevInfo di;
  if (!device_info(di)) return CKL_ERR_CUDA;
  if (di.major != 10) return CKL_ERR_UNSUPPORTED;
  if (!encode_fn()) return CKL_ERR_CUDA;
  uint8_t* w8 = static_cast<uint8_t*>(static_scratch_ptr());
  if (!w8) return CKL_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The buffer still holds the previous call's words: the header is cleared
  // before the prep, exactly as in ckl_forward, and the GEMM and combine
  // overwrite every other word they read.
  int rc = clear_and_prep(topk_idx, topk_logp, mask, T, K, V, w8, L, st, nullptr);
  if (rc != CKL_OK) return rc;
  rc = forward_gemm_combine<false>(H, W, mask, T, d, V, K, loss, lse, w8, L, di, st, nullptr);
  if (rc != CKL_OK) return rc;
  if (device_status) {
    Header* hdr = reinterpret_cast<Header*>(w8);
    copy_status_kernel<<<1, 1, 0, st>>>(&hdr->status, device_status);
    if (cudaGetLastError() != cudaSuccess) return CKL_ERR_CUDA;
  }
  return CKL_OK;
}

}  // extern "C"
