// C ABI of libqnf4 (declared in include/qnf4.h): argument checks, workspace
// layout, tensor-map creation and kernel launches. All device code of the library
// is compiled in this one translation unit.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cublas_v2.h>
#include <cusolverDn.h>
#include <dlfcn.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/qnf4.h"
#include "chanq.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "gemm.cuh"
#include "loftq.cuh"
#include "quant.cuh"
#include "tables.h"

namespace qnf4 {
namespace {

thread_local std::string g_last = "";
unsigned long long g_wait_ns = 1000000000ull;

qnf4_status fail(qnf4_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last = buf;
  return s;
}
qnf4_status ok() { return QNF4_OK; }

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::atomic<unsigned long long> g_launches{0};
thread_local cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;

// Check the last launch(es) and count `n` kernels of this library as launched.
// first failure of a cudaLaunchKernelEx launch since the last launched() check
thread_local cudaError_t g_launch_err = cudaSuccess;

qnf4_status launched(const char* what, int n = 1) {
  g_launches.fetch_add(static_cast<unsigned long long>(n), std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = g_launch_err;
  g_launch_err = cudaSuccess;
  if (e != cudaSuccess) return fail(QNF4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return QNF4_OK;
}

// Launch as a programmatic dependent of the previous kernel in the stream: the kernel
// may start (and run its prologue) while that kernel finishes; every kernel launched
// this way calls griddepcontrol.wait before it touches global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess && g_launch_err == cudaSuccess) g_launch_err = e;
  return e;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::mutex mu;
  static std::vector<int> cache;
  std::lock_guard<std::mutex> lk(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 148;
  }
  return cache[dev];
}

QuantTab make_tab() {
  const Nf4Tables& t = nf4_tables();
  QuantTab q;
  std::memcpy(q.thr, t.thr, sizeof(q.thr));
  std::memcpy(q.levels, t.levels, sizeof(q.levels));
  q.bin_h = t.bin_h;
  std::memcpy(q.bin_th, t.bin_th, sizeof(q.bin_th));
  return q;
}

int quant_grid_chunks(int64_t chunks) {
  // persistent: kQCtasPerSm streaming CTAs per SM, never more warps than chunks
  const int64_t ctas = (chunks + kQWorkers - 1) / kQWorkers;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ctas, num_sms() * kQCtasPerSm)));
}
int quant_grid(int64_t nblocks) { return quant_grid_chunks((nblocks + kQChunkBlocks - 1) / kQChunkBlocks); }

bool g_quant_smem_set[64] = {};

qnf4_status quant_smem_attr() {
  // the quantizer's code search needs the bin table (always found for the NF4 levels)
  if (nf4_tables().bin_h < 1 || nf4_tables().bin_h > kQMaxH)
    return fail(QNF4_ERR_ARG, "internal: no NF4 bin table the quantizer can hold");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !g_quant_smem_set[dev]) {
    for (auto fn : {k_nf4_quant<true, true>, k_nf4_quant<true, false>, k_nf4_quant<false, true>,
                    k_nf4_quant<false, true, true>}) {
      const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(kQSmem));
      if (e != cudaSuccess) return fail(QNF4_ERR_CUDA, "smem attribute: %s", cudaGetErrorString(e));
    }
    g_quant_smem_set[dev] = true;
  }
  return QNF4_OK;
}

qnf4_status check_weight(const qnf4_weight* w) {
  if (!w) return fail(QNF4_ERR_ARG, "weight is NULL");
  if (w->block1 != 64 || w->block2 != 256)
    return fail(QNF4_ERR_ARG, "block1 must be 64 and block2 256 (got %d, %d)", w->block1, w->block2);
  if (w->N <= 0 || w->K <= 0) return fail(QNF4_ERR_SHAPE, "N and K must be positive");
  if (w->K % 64) return fail(QNF4_ERR_SHAPE, "K must be a multiple of 64 (got %lld)", (long long)w->K);
  if (!w->packed || !w->code2 || !w->scale2 || !w->mean) return fail(QNF4_ERR_ARG, "weight has a NULL buffer");
  if (!al16(w->packed) || !al16(w->code2) || !al16(w->scale2) || !al16(w->mean))
    return fail(QNF4_ERR_ALIGN, "weight buffers must be 16-byte aligned");
  return ok();
}


// ---------------------------------------------------------------------------
// tcgen05 GEMM planning: tile sizes, split-K and the workspace carve-up
// ---------------------------------------------------------------------------
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// 2-D tensor map over a row-major [outer, inner] matrix with row stride ld elements.
bool make_map(CUtensorMap* m, const void* ptr, bool u8, uint64_t inner, uint64_t outer,
              uint64_t ld, uint32_t box_in, uint32_t box_out, bool sw128) {
  std::memset(m, 0, sizeof(*m));
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = u8 ? 1 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * es};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The quantizer's view of a weight: a [nblocks, 64] bf16 matrix, loaded in boxes of
// kQChunkBlocks rows with the 128-byte swizzle.
bool quant_map(CUtensorMap* m, const void* W, int64_t nblocks) {
  if (nblocks > INT32_MAX) return false;  // the row coordinate is a 32-bit integer
  return make_map(m, W, false, 64, static_cast<uint64_t>(nblocks), 64, 64, kQChunkBlocks, true);
}

// One weight as the only job of a quantize launch (false if its map cannot be made).
bool one_quant_job(QuantJobs* j, const void* W, int64_t nblocks, uint8_t* packed, float* absmax) {
  std::memset(j, 0, sizeof(*j));
  j->n = 1;
  j->nblocks[0] = nblocks;
  j->chunk0[0] = 0;
  j->chunk0[1] = (nblocks + kQChunkBlocks - 1) / kQChunkBlocks;
  j->packed[0] = reinterpret_cast<uint32_t*>(packed);
  j->absmax[0] = absmax;
  return quant_map(&j->map[0], W, nblocks);
}

// CTAs of a double-quantization launch over nb2 256-blocks, each a contiguous run.
int dq_grid(DqJobs* d, int64_t nb2) {
  const int64_t P = std::max<int64_t>(1, std::min<int64_t>((nb2 + 7) / 8, num_sms() * 4));
  d->per_cta = std::max<int64_t>(1, (nb2 + P - 1) / P);
  return static_cast<int>(std::max<int64_t>(1, (nb2 + d->per_cta - 1) / d->per_cta));
}

// One tensor as the only job of a double-quantization launch; returns the grid.
int one_dq_job(DqJobs* d, const float* c, int64_t nb1, const double* part, int npart, int64_t count,
               uint8_t* code2, float* scale2, float* mean, const double* sse_part, int nsse,
               double* sse_out) {
  std::memset(d, 0, sizeof(*d));
  d->n = 1;
  d->c[0] = c;
  d->nb1[0] = nb1;
  d->count[0] = count;
  d->part[0] = part;
  d->npart = npart;
  d->code2[0] = code2;
  d->scale2[0] = scale2;
  d->mean[0] = mean;
  d->sse_part[0] = sse_part;
  d->nsse = nsse;
  d->sse_out[0] = sse_out;
  d->b2_0[0] = 0;
  d->b2_0[1] = (nb1 + 255) / 256;
  return dq_grid(d, d->b2_0[1]);
}

// x [M, K] bf16 seen as [K/64][M][64]: box = 16 column blocks x rows x 64 columns
// (128-byte swizzle on the 128-byte rows).
bool make_map_xblocks(CUtensorMap* m, const void* x, uint64_t K, uint64_t M, uint32_t rows) {
  std::memset(m, 0, sizeof(*m));
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, M, K / 64};
  cuuint64_t strides[2] = {K * 2, 128};
  cuuint32_t box[3] = {64, rows, kDecSbBlocks};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// packed [N, K/2] bytes seen as [N][K/256][128] (K a multiple of 256): box = rows x 4
// column groups x 128 bytes, each row's 512 bytes in order (128-byte swizzle).
bool make_map_wcols(CUtensorMap* m, const void* packed, uint64_t K, uint64_t N, uint32_t rows) {
  std::memset(m, 0, sizeof(*m));
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, K / 256, N};
  cuuint64_t strides[2] = {128, K / 2};
  cuuint32_t box[3] = {128, kDecGroups, rows};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(packed), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct GemmPlan {
  int asrc = 0, tn = 16, has_ext = 0;
  int64_t rows = 0, cols = 0;
  int nsteps = 0, row_tiles = 0, col_tiles = 0, s1 = 1, s2 = 0;
  // work units: full_tiles whole tiles, then tail_tiles tiles cut into tail_splits
  // contraction slices of tail_sps steps; grid = persistent CTAs
  int full_tiles = 0, tail_tiles = 0, tail_splits = 1, tail_sps = 0, units = 0, grid = 1;
  int ctas_per_sm = 1;
  int nset = 1;  // converter warp sets (4 warps each)
  int lut = 0;   // NF4 dequantization through the shared-memory pair table
  size_t smem = 0;
  size_t part_floats() const {
    return tail_splits > 1 ? static_cast<size_t>(tail_tiles) * tail_splits * tn * 128 : 0;
  }
  int64_t tiles() const { return static_cast<int64_t>(row_tiles) * col_tiles; }
};

constexpr size_t kSmemLimit = 227 * 1024;

// Tiling (measured on the Llama shapes): three converter sets for wide tiles, one set
// and two CTAs per SM for thin tiles, a 7-deep TMEM A ring for thin tiles, and
// contraction slices of at least four steps.
constexpr int kNsetWide = 3;
constexpr int kNsetThin = 1;
constexpr int kCtasThin = 2;
constexpr int kS2ThinTmem = 7;
constexpr int kMinSplitSteps = 4;

int tn_for_tokens(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  return 256;
}

GemmPlan plan_gemm(int asrc, int64_t rows, int64_t cols, int64_t contraction, int tn,
                   int has_ext, int nsm) {
  GemmPlan p;
  p.asrc = asrc;
  p.tn = tn;
  p.has_ext = has_ext;
  p.rows = rows;
  p.cols = cols;
  p.nsteps = static_cast<int>((contraction + kStep - 1) / kStep);
  p.row_tiles = static_cast<int>((rows + kRowsTile - 1) / kRowsTile);
  p.col_tiles = static_cast<int>((cols + tn - 1) / tn);
  // Thin N tiles (decode, rank-r GEMMs) are latency bound: give them two CTAs per SM
  // and a shallower dequant ring; wide tiles take the whole shared memory.
  const bool thin = tn <= 32;
  p.ctas_per_sm = thin ? kCtasThin : 1;
  // Wide tiles need several converter sets to keep the tensor core fed; thin tiles
  // run more CTAs per SM instead.
  p.nset = src_deq(asrc) ? (thin ? kNsetThin : kNsetWide) : 1;
  if (src_tmem_a(asrc)) {
    // TMEM A stages. Each is reusable only after the MMA that read it has completed,
    // so the ring depth bounds the steps in flight per MMA round trip: as deep as the
    // accumulator leaves room for (256 columns per CTA at two CTAs per SM, 512 at one).
    const int room = static_cast<int>(((p.ctas_per_sm == 2 ? 256u : 512u) - acc_cols(tn)) / 32u);
    p.s2 = std::min(room, thin ? kS2ThinTmem : 8);
    if (p.s2 > kMaxS2) p.s2 = kMaxS2;
  } else {
    p.s2 = src_deq(asrc) ? ((thin ? 2 : 4)) : 0;
  }
  // Thin NF4 tiles (decode) dequantize through the shared-memory pair table (32 copies):
  // their converters are bound by integer issue, which the table moves to the load and
  // fma pipes.
  const bool nf4 = asrc == A_NF4_K || asrc == A_NF4_MN;
  p.lut = (nf4 && thin) ? 32 : 0;
  // 1 KB to align the dynamic buffer, 1 KB for static shared data, per CTA
  const size_t budget = (p.ctas_per_sm == 2 ? (kSmemLimit / 2 - 2048) : kSmemLimit) - 2048;
  for (int pass = 0; pass < 2; ++pass) {
    const SmemPlan one = smem_plan(asrc, tn, 1, p.s2, has_ext, p.lut);
    const size_t fixed = one.total - one.slot1;
    p.s1 = static_cast<int>(std::min<size_t>(kMaxS1, (budget - fixed) / one.slot1));
    // the dequantized-A ring may not be deeper than the load ring (its stages are
    // released through the load ring's barriers)
    if (p.s2 > p.s1) p.s2 = p.s1;
  }
  p.smem = smem_plan(asrc, tn, p.s1, p.s2, has_ext, p.lut).total + 1024;
  // Persistent CTAs, one per slot, take the tiles in waves. The tiles of a last,
  // partial wave are cut into contraction slices so that wave is as full as it can
  // be: as many slices as the idle slots allow, at least four steps each (each slice
  // costs a partial tile and one more term in the last slice's reduction).
  const int64_t tiles = p.tiles();
  const int64_t slots = static_cast<int64_t>(nsm) * p.ctas_per_sm;
  p.full_tiles = static_cast<int>((tiles / slots) * slots);
  p.tail_tiles = static_cast<int>(tiles - p.full_tiles);
  int best = 1;
  if (p.tail_tiles > 0 && p.nsteps > 1) {
    const int max_splits = std::max(1, p.nsteps / kMinSplitSteps);
    best = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(max_splits, slots / p.tail_tiles)));
  }
  p.tail_sps = (p.nsteps + best - 1) / best;
  p.tail_splits = p.tail_sps > 0 ? (p.nsteps + p.tail_sps - 1) / p.tail_sps : 1;
  p.units = p.full_tiles + p.tail_tiles * p.tail_splits;
  p.grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(p.units, slots)));
  return p;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace of one linear-layer call (forward or backward).
struct LinPlan {
  int r16 = 16;
  int64_t ldm = 0, ldn = 0;
  GemmPlan u, v, main, da, db;
  size_t off_up = 0, off_ut = 0, off_vp = 0, off_vt = 0, off_bt = 0, off_part = 0, off_cnt = 0;
  size_t off_upart = 0, off_ucnt = 0;  // the u kernel's own split-K area (it may overlap the next)
  size_t total = 0;
};

LinPlan plan_linear(int main_src, int64_t N, int64_t K, int64_t M, int r, bool bwd, int nsm) {
  LinPlan L;
  L.r16 = ((r + 15) / 16) * 16;
  L.ldm = ((M + 7) / 8) * 8;
  L.ldn = ((N + 7) / 8) * 8;
  const int tnm = tn_for_tokens(M);
  size_t part = 0;
  int64_t cnt = 1;
  L.u = plan_gemm(A_DENSE_K, M, L.r16, K, L.r16, 0, nsm);
  if (!bwd) {
    L.main = plan_gemm(main_src, N, M, K, tnm, 1, nsm);
  } else {
    L.v = plan_gemm(A_DENSE_K, M, L.r16, N, L.r16, 0, nsm);
    L.main = plan_gemm(main_src, K, M, N, tnm, 1, nsm);
    L.da = plan_gemm(A_DENSE_MN, K, L.r16, M, L.r16, 0, nsm);
    L.db = plan_gemm(A_DENSE_MN, N, L.r16, M, L.r16, 0, nsm);
    for (const GemmPlan* g : {&L.v, &L.da, &L.db}) {
      part = std::max(part, g->part_floats());
      cnt = std::max(cnt, g->tiles());
    }
  }
  part = std::max(part, L.main.part_floats());
  cnt = std::max(cnt, L.main.tiles());
  size_t o = 0;
  L.off_up = o;
  o = align256(o + static_cast<size_t>(M) * 64 * 2);
  if (bwd) {
    L.off_ut = o;
    o = align256(o + static_cast<size_t>(L.r16) * L.ldm * 2);
    L.off_vp = o;
    o = align256(o + static_cast<size_t>(M) * 64 * 2);
    L.off_vt = o;
    o = align256(o + static_cast<size_t>(L.r16) * L.ldm * 2);
    L.off_bt = o;
    o = align256(o + static_cast<size_t>(L.r16) * L.ldn * 2);
  }
  L.off_upart = o;
  o = align256(o + L.u.part_floats() * sizeof(float));
  L.off_part = o;
  o = align256(o + part * sizeof(float));
  // counters last, so one memset clears both areas
  L.off_ucnt = o;
  o = align256(o + static_cast<size_t>(L.u.tiles()) * sizeof(unsigned int));
  L.off_cnt = o;
  o = align256(o + static_cast<size_t>(cnt) * sizeof(unsigned int));
  L.total = o;
  return L;
}

bool g_smem_set[6][4][3][64] = {};

template <int ASRC, int NSET, int MINB>
qnf4_status launch_gemm(const GemmPlan& p, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& bx, const CUtensorMap& o, const CUtensorMap& t, GemmArgs g,
                        cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !g_smem_set[ASRC][NSET][MINB][dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_gemm<ASRC, NSET, MINB>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(kSmemLimit - 1024));
    if (e != cudaSuccess) return fail(QNF4_ERR_CUDA, "smem attribute: %s", cudaGetErrorString(e));
    g_smem_set[ASRC][NSET][MINB][dev] = true;
  }
  if (p.s1 < 1 || p.s1 > kMaxS1 || p.s2 < 0 || p.s2 > kMaxS2 || p.s2 > p.s1 || p.tn < 16 || p.tn > 256 ||
      p.tn % 16 || tmem_cols(ASRC, p.tn, p.s2) > (p.ctas_per_sm == 2 ? 256u : 512u) ||
      (src_deq(ASRC) && NSET > p.s2))
    return fail(QNF4_ERR_ARG, "internal tiling out of range (s1 %d, s2 %d, tn %d)", p.s1, p.s2, p.tn);
  g.rows = p.rows;
  g.cols = p.cols;
  g.nsteps = p.nsteps;
  g.row_tiles = p.row_tiles;
  g.full_tiles = p.full_tiles;
  g.tail_tiles = p.tail_tiles;
  g.tail_splits = p.tail_splits;
  g.tail_sps = p.tail_sps;
  g.nunits = p.units;
  g.tn = p.tn;
  g.s1 = p.s1;
  g.s2 = p.s2;
  g.has_ext = p.has_ext;
  g.lut = p.lut;
  g.part_elems = static_cast<int64_t>(p.part_floats());
  g.cnt_elems = p.tail_tiles;
  g.wait_ns = g_wait_ns;
  if (!p.has_ext) g.stage = 0;  // the staging buffers live in the adapter tile
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  if (p.units < 1) return QNF4_OK;  // empty D: nothing to compute
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.blockDim = dim3(gemm_threads(NSET), 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_gemm<ASRC, NSET, MINB>, a, b, bx, o, t, g);
  if (e != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaGetLastError();
    return fail(QNF4_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(e));
  }
  return launched("gemm");
}

// The instantiated (source, converter sets, CTAs per SM) combinations.
template <int ASRC>
qnf4_status launch_deq(const GemmPlan& p, const CUtensorMap& a, const CUtensorMap& b,
                       const CUtensorMap& bx, const CUtensorMap& o, const CUtensorMap& t,
                       const GemmArgs& g, cudaStream_t s) {
  const int key = p.nset * 10 + p.ctas_per_sm;
  switch (key) {
    case 11: return launch_gemm<ASRC, 1, 1>(p, a, b, bx, o, t, g, s);
    case 12: return launch_gemm<ASRC, 1, 2>(p, a, b, bx, o, t, g, s);
    case 21: return launch_gemm<ASRC, 2, 1>(p, a, b, bx, o, t, g, s);
    case 22: return launch_gemm<ASRC, 2, 2>(p, a, b, bx, o, t, g, s);
    case 31: return launch_gemm<ASRC, 3, 1>(p, a, b, bx, o, t, g, s);
    default: return fail(QNF4_ERR_ARG, "no kernel for %d converter sets x %d CTAs/SM", p.nset, p.ctas_per_sm);
  }
}

qnf4_status launch_any(const GemmPlan& p, const CUtensorMap& a, const CUtensorMap& b,
                       const CUtensorMap& bx, const CUtensorMap& o, const CUtensorMap& t,
                       const GemmArgs& g, cudaStream_t s) {
  switch (p.asrc) {
    case A_NF4_K: return launch_deq<A_NF4_K>(p, a, b, bx, o, t, g, s);
    case A_NF4_MN: return launch_deq<A_NF4_MN>(p, a, b, bx, o, t, g, s);
    case A_DENSE_K:
      return p.ctas_per_sm == 2 ? launch_gemm<A_DENSE_K, 1, 2>(p, a, b, bx, o, t, g, s)
                                : launch_gemm<A_DENSE_K, 1, 1>(p, a, b, bx, o, t, g, s);
    case A_DENSE_MN:
      return p.ctas_per_sm == 2 ? launch_gemm<A_DENSE_MN, 1, 2>(p, a, b, bx, o, t, g, s)
                                : launch_gemm<A_DENSE_MN, 1, 1>(p, a, b, bx, o, t, g, s);
    case A_CHANQ_MN: return launch_deq<A_CHANQ_MN>(p, a, b, bx, o, t, g, s);
    default: return launch_deq<A_CHANQ_K>(p, a, b, bx, o, t, g, s);
  }
}

GemmArgs base_args() {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  const Nf4Tables& t = nf4_tables();
  std::memcpy(g.levels, t.levels, sizeof(g.levels));
  // extents for the checked build's index tests: unbounded until a caller narrows them
  g.out_elems = g.out2_elems = g.part_elems = g.cnt_elems = g.cst_elems = INT64_MAX;
  return g;
}

// The frozen base of one linear layer, in one of its three storage forms.
struct BaseSrc {
  int kind = A_NF4_K;        // A_NF4_K (NF4), A_DENSE_K (bf16), A_CHANQ_K (per-channel)
  const qnf4_weight* w = nullptr;
  const void* Wd = nullptr;  // dense bf16 [N, K]
  const uint8_t* cq_packed = nullptr;
  const int64_t* cq_row_off = nullptr;
  const uint8_t* cq_bits = nullptr;
  const float* cq_map = nullptr;
  const int64_t* cq_map_off = nullptr;
  const float* cq_absmax = nullptr;
  // per-channel backward: the codes widened to the NF4 nibble layout [N, K/2] and the
  // rows' 16-entry tables [N, 16], made in the workspace by k_chanq_widen
  uint8_t* cq_wide = nullptr;
  float* cq_tab = nullptr;
  int64_t N = 0, K = 0;
};

// Output map of the staged epilogue: bf16 D with rows contiguous (ld elements between
// columns), stored in boxes of 128 rows x 8 columns. False when the layout does not allow
// it (row stride not a multiple of 16 bytes); the epilogue then stores element by element.
bool stage_map(CUtensorMap* m, void* out, int64_t rows, int64_t cols, int64_t ld) {
  std::memset(m, 0, sizeof(*m));
  if ((ld * 2) % 16 != 0 || !al16(out)) return false;
  return make_map(m, out, false, rows, cols, ld, 128, 8, false);
}

// Workspace after the backward's own: the widened codes [N, K/2] and the tables [N, 16].
size_t chanq_wide_bytes(int64_t N, int64_t K) {
  return align256(static_cast<size_t>(N) * static_cast<size_t>(K / 2)) +
         align256(static_cast<size_t>(N) * 16 * sizeof(float));
}

// 2-D fp32 tensor [outer, inner] (row stride ld elements), no swizzle.
bool make_map_f32(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld,
                  uint32_t box_in, uint32_t box_out) {
  std::memset(m, 0, sizeof(*m));
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

qnf4_status map_fail() { return fail(QNF4_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or refused the layout"); }

// u = x A^T (contraction K), written as bf16(scale u) into up [M, 64] and, when ut is
// given, transposed into ut [r16, ldm].
qnf4_status run_u(const LinPlan& L, const void* x, const void* A, int64_t M, int64_t K, int r,
                  float scale, uint16_t* up, uint16_t* ut, float* part, unsigned* cnt, cudaStream_t s) {
  CUtensorMap ma, mb, none;
  std::memset(&none, 0, sizeof(none));
  if (!make_map(&ma, x, false, K, M, K, 64, 128, true)) return map_fail();
  if (!make_map(&mb, A, false, K, r, K, 64, L.r16, true)) return map_fail();
  GemmArgs g = base_args();
  g.epi = EPI_UV;
  g.out = up;
  g.out2 = ut;
  g.o2_ld = L.ldm;
  g.out_elems = M * 64;
  g.out2_elems = static_cast<int64_t>(L.r16) * L.ldm;
  g.scale = scale;
  g.part = part;
  g.counters = cnt;
  return launch_any(L.u, ma, mb, none, none, none, g, s);
}

// ---------------------------------------------------------------------------
// Decode-size forward (M <= 16 tokens): k_lora_u, then k_nf4_decode (see decode.cuh)
// ---------------------------------------------------------------------------
constexpr int64_t kDecodeMaxTokens = 16;

// Workspace of one decode-size layer: its adapter projection partials, 256-aligned.
size_t decode_ws_bytes(int64_t K, int64_t M, int r) {
  const int64_t ks = (K + kDecUChunk - 1) / kDecUChunk;
  return align256(static_cast<size_t>(ks) * r * M * sizeof(float));
}

bool g_dec_smem_set[2][64] = {};

template <int Q>
cudaError_t launch_decode(const DecodeArgs& a, int P, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !g_dec_smem_set[Q - 1][dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k_nf4_decode<Q>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(kDecSmem));
    if (e != cudaSuccess) return e;
    g_dec_smem_set[Q - 1][dev] = true;
  }
  return launch_pdl(k_nf4_decode<Q>, dim3(P), dim3(kDecBlockThreads), kDecSmem, s, a, g_wait_ns);
}

// Decode-size forward of n independent layers in one launch pair (k_lora_u, then
// k_nf4_decode); the layers share M, r and scale. Arguments are checked by the caller.
qnf4_status decode_group(int n, const qnf4_weight* w, const void* const* xs, int64_t M,
                         const void* const* As, const void* const* Bs, int r, float scale,
                         void* const* hs, void* ws, size_t ws_bytes, cudaStream_t s) {
  static thread_local DecodeArgs a;  // about 10 KB: kept off the stack
  std::memset(&a, 0, sizeof(a));
  a.n = n;
  a.M = static_cast<int>(M);
  a.r = r;
  a.scale = scale;
  std::memcpy(a.levels, nf4_tables().levels, sizeof(a.levels));
  size_t need = 0;
  int64_t units = 0, kmax = 0;
  double total = 0.0;  // work = units x K (bytes per unit are 8 K)
  for (int l = 0; l < n; ++l) {
    const int64_t N = w[l].N, K = w[l].K;
    DecLayer& L = a.L[l];
    L.N = N;
    L.K = K;
    L.nkb = static_cast<int>(K / 64);
    L.ks = static_cast<int>((K + kDecUChunk - 1) / kDecUChunk);
    L.w3d = K % 256 == 0 ? 1 : 0;
    L.unit0 = units;
    L.nb2 = (N * (K / 64) + 255) / 256;
    L.code2 = w[l].code2;
    L.scale2 = w[l].scale2;
    L.mean = w[l].mean;
    L.x = static_cast<const uint16_t*>(xs[l]);
    L.A = static_cast<const uint16_t*>(As[l]);
    L.Bm = static_cast<const uint16_t*>(Bs[l]);
    L.h = static_cast<uint16_t*>(hs[l]);
    L.upart = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + need);
    need += decode_ws_bytes(K, M, r);
    for (int i = 0; i < kDecMaxRb; ++i) {
      const uint32_t rows = 16u * (i + 1);
      const bool ok = L.w3d ? make_map_wcols(&a.wmap[l][i], w[l].packed, K, N, rows)
                            : make_map(&a.wmap[l][i], w[l].packed, true, K / 2, N, K / 2, 128, rows, true);
      if (!ok) return map_fail();
    }
    if (!make_map_xblocks(&a.xmap[l], xs[l], K, M, static_cast<uint32_t>(M))) return map_fail();
    const int64_t rbs = (N + 15) / 16;
    units += rbs;
    total += static_cast<double>(rbs) * static_cast<double>(K);
    kmax = std::max(kmax, K);
  }
  if (!ws || ws_bytes < need) return fail(QNF4_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, need);
  a.units = units;
  // CTA p takes the units from the first one whose start lies at or past p / P of the
  // total work (units x K), so every CTA streams about the same number of bytes
  const int P = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({num_sms(), units, kDecMaxCta})));
  {
    int p = 0;
    double cum = 0.0;
    int64_t u = 0;
    a.cta_unit[0] = 0;
    for (int l = 0; l < n; ++l) {
      const int64_t rbs = (w[l].N + 15) / 16;
      for (int64_t b = 0; b < rbs; ++b, ++u) {
        while (p + 1 < P && cum >= total * (p + 1) / P) a.cta_unit[++p] = u;
        cum += static_cast<double>(w[l].K);
      }
    }
    while (p < P) a.cta_unit[++p] = units;
  }
  if (g_ev_start) cudaEventRecord(g_ev_start, s);
  const int ksmax = static_cast<int>((kmax + kDecUChunk - 1) / kDecUChunk);
  cudaError_t e = launch_pdl(k_lora_u, dim3(r, ksmax, n), dim3(128), 0, s, a);
  if (e != cudaSuccess) return fail(QNF4_ERR_CUDA, "k_lora_u launch: %s", cudaGetErrorString(e));
  e = M <= 8 ? launch_decode<1>(a, P, s) : launch_decode<2>(a, P, s);
  if (e != cudaSuccess) return fail(QNF4_ERR_CUDA, "k_nf4_decode launch: %s", cudaGetErrorString(e));
  if (g_ev_stop) cudaEventRecord(g_ev_stop, s);
  return launched("decode_fwd", 2);
}

qnf4_status decode_fwd(const qnf4_weight* w, const void* x, int64_t M, const void* A, const void* B,
                       int r, float scale, void* h, void* ws, size_t ws_bytes, cudaStream_t s) {
  return decode_group(1, w, &x, M, &A, &B, r, scale, &h, ws, ws_bytes, s);
}

qnf4_status linear_fwd(const BaseSrc& src, const void* x, int64_t M, const void* A, const void* B,
                       int r, float scale, void* h, void* ws, size_t ws_bytes, cudaStream_t s) {
  const int64_t N = src.N, K = src.K;
  const LinPlan L = plan_linear(src.kind, N, K, M, r, false, num_sms());
  if (!ws || ws_bytes < L.total) return fail(QNF4_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, L.total);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  uint16_t* up = reinterpret_cast<uint16_t*>(w8 + L.off_up);
  float* part = reinterpret_cast<float*>(w8 + L.off_part);
  unsigned* cnt = reinterpret_cast<unsigned*>(w8 + L.off_cnt);
  if (cudaMemsetAsync(w8 + L.off_ucnt, 0, L.total - L.off_ucnt, s) != cudaSuccess)
    return launched("memset", 0);
  qnf4_status st = run_u(L, x, A, M, K, r, scale, up, nullptr,
                         reinterpret_cast<float*>(w8 + L.off_upart),
                         reinterpret_cast<unsigned*>(w8 + L.off_ucnt), s);
  if (st != QNF4_OK) return st;
  CUtensorMap ma, mb, mbx, none;
  std::memset(&none, 0, sizeof(none));
  std::memset(&ma, 0, sizeof(ma));
  const int tn = L.main.tn;
  if (src.kind == A_NF4_K) {
    if (!make_map(&ma, src.w->packed, true, K / 2, N, K / 2, 32, 128, false)) return map_fail();
  } else if (src.kind == A_DENSE_K) {
    if (!make_map(&ma, src.Wd, false, K, N, K, 64, 128, true)) return map_fail();
  }
  if (!make_map(&mb, x, false, K, M, K, 64, tn, true)) return map_fail();
  if (!make_map(&mbx, up, false, 64, M, 64, 64, tn, true)) return map_fail();
  GemmArgs g = base_args();
  g.ext_k16 = L.r16 / 16;
  g.ext_r = r;
  g.ext_a = static_cast<const uint16_t*>(B);
  g.ext_ld = r;
  g.wN = N;
  g.nbk = K / 64;
  if (src.kind == A_NF4_K) {
    g.code2 = src.w->code2;
    g.scale2 = src.w->scale2;
    g.mean = src.w->mean;
    g.packed = src.w->packed;
  } else if (src.kind == A_CHANQ_K) {
    g.cq_packed = src.cq_packed;
    g.cq_row_off = src.cq_row_off;
    g.cq_bits = src.cq_bits;
    g.cq_map = src.cq_map;
    g.cq_map_off = src.cq_map_off;
    g.cq_absmax = src.cq_absmax;
  }
  g.epi = EPI_BF16;
  g.out = h;
  g.o_rs = 1;
  g.o_cs = N;
  g.out_elems = M * N;
  if (src.kind == A_NF4_K) g.cst_elems = N * (K / 64);
  CUtensorMap mo;
  g.stage = stage_map(&mo, h, N, M, N) ? 1 : 0;
  g.part = part;
  g.counters = cnt;
  g.lazy_dep = 1;  // only the adapter chunk reads what the u kernel writes
  if (g_ev_start) cudaEventRecord(g_ev_start, s);
  st = launch_any(L.main, ma, mb, mbx, mo, none, g, s);
  if (g_ev_stop) cudaEventRecord(g_ev_stop, s);
  return st;
}

qnf4_status linear_bwd(const BaseSrc& src, const void* x, const void* dY, int64_t M, const void* A,
                       const void* B, int r, float scale, void* dX, float* dA, float* dB, void* ws,
                       size_t ws_bytes, cudaStream_t s) {
  const int64_t N = src.N, K = src.K;
  const int main_src =
      src.kind == A_NF4_K ? A_NF4_MN : (src.kind == A_CHANQ_K ? A_CHANQ_MN : A_DENSE_MN);
  const LinPlan L = plan_linear(main_src, N, K, M, r, true, num_sms());
  if (!ws || ws_bytes < L.total) return fail(QNF4_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, L.total);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  uint16_t* ut = reinterpret_cast<uint16_t*>(w8 + L.off_ut);
  uint16_t* vp = reinterpret_cast<uint16_t*>(w8 + L.off_vp);
  uint16_t* vt = reinterpret_cast<uint16_t*>(w8 + L.off_vt);
  uint16_t* bt = reinterpret_cast<uint16_t*>(w8 + L.off_bt);
  float* part = reinterpret_cast<float*>(w8 + L.off_part);
  unsigned* cnt = reinterpret_cast<unsigned*>(w8 + L.off_cnt);
  if (cudaMemsetAsync(w8 + L.off_ucnt, 0, L.total - L.off_ucnt, s) != cudaSuccess)
    return launched("memset", 0);
  // B^T for v = dY B
  {
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((N * r + 255) / 256, num_sms() * 4)));
    k_transpose_b<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(B), N, r, bt, L.ldn);
    qnf4_status st = launched("transpose_b");
    if (st != QNF4_OK) return st;
  }
  qnf4_status st = QNF4_OK;
  CUtensorMap none;
  std::memset(&none, 0, sizeof(none));
  // Order: v and u, then dA and dB while x and dY are still in L2 (both are
  // HBM-bound), then dX (tensor-bound).
  // v = dY B  ->  vp = bf16(scale v) [M, 64], vt = its transpose [r16, ldm]
  {
    CUtensorMap ma, mb;
    if (!make_map(&ma, dY, false, N, M, N, 64, 128, true)) return map_fail();
    if (!make_map(&mb, bt, false, N, r, L.ldn, 64, L.r16, true)) return map_fail();
    GemmArgs g = base_args();
    g.epi = EPI_UV;
    g.out = vp;
    g.out2 = vt;
    g.o2_ld = L.ldm;
    g.out_elems = M * 64;
    g.out2_elems = static_cast<int64_t>(L.r16) * L.ldm;
    g.scale = scale;
    g.part = part;
    g.counters = cnt;
    st = launch_any(L.v, ma, mb, none, none, none, g, s);
    if (st != QNF4_OK) return st;
  }
  // (scale u)^T for dB
  st = run_u(L, x, A, M, K, r, scale, nullptr, ut,
                         reinterpret_cast<float*>(w8 + L.off_upart),
                         reinterpret_cast<unsigned*>(w8 + L.off_ucnt), s);
  if (st != QNF4_OK) return st;
  // dA = (scale v)^T x  -> [r, K]
  {
    CUtensorMap ma, mb;
    if (!make_map(&ma, x, false, K, M, K, 64, 64, true)) return map_fail();
    if (!make_map(&mb, vt, false, M, L.r16, L.ldm, 64, L.r16, true)) return map_fail();
    GemmArgs g = base_args();
    g.epi = EPI_F32;
    g.out = dA;
    g.o_rs = 1;
    g.o_cs = K;
    g.out_cols = r;
    g.out_elems = static_cast<int64_t>(r) * K;
    g.scale = 1.f;
    g.part = part;
    g.counters = cnt;
    st = launch_any(L.da, ma, mb, none, none, none, g, s);
    if (st != QNF4_OK) return st;
  }
  // dB = dY^T (scale u)  -> [N, r]
  {
    CUtensorMap ma, mb;
    if (!make_map(&ma, dY, false, N, M, N, 64, 64, true)) return map_fail();
    if (!make_map(&mb, ut, false, M, L.r16, L.ldm, 64, L.r16, true)) return map_fail();
    GemmArgs g = base_args();
    g.epi = EPI_F32;
    g.out = dB;
    g.o_rs = r;
    g.o_cs = 1;
    g.out_cols = r;
    g.out_elems = N * r;
    g.scale = 1.f;
    g.part = part;
    g.counters = cnt;
    st = launch_any(L.db, ma, mb, none, none, none, g, s);
    if (st != QNF4_OK) return st;
  }
  // dX = dY W_hat + (scale v) A
  {
    CUtensorMap ma, mb, mbx, mt;
    std::memset(&mt, 0, sizeof(mt));
    const int tn = L.main.tn;
    if (main_src == A_NF4_MN) {
      if (!make_map(&ma, src.w->packed, true, K / 2, N, K / 2, 64, 64, false)) return map_fail();
    } else if (main_src == A_CHANQ_MN) {
      if (!make_map(&ma, src.cq_wide, true, K / 2, N, K / 2, 64, 64, false)) return map_fail();
      if (!make_map_f32(&mt, src.cq_tab, 16, N, 16, 16, 64)) return map_fail();
    } else {
      if (!make_map(&ma, src.Wd, false, K, N, K, 64, 64, true)) return map_fail();
    }
    if (!make_map(&mb, dY, false, N, M, N, 64, tn, true)) return map_fail();
    if (!make_map(&mbx, vp, false, 64, M, 64, 64, tn, true)) return map_fail();
    GemmArgs g = base_args();
    g.ext_k16 = L.r16 / 16;
    g.ext_r = r;
    g.ext_a = static_cast<const uint16_t*>(A);
    g.ext_ld = K;
    g.wN = N;
    g.nbk = K / 64;
    if (main_src == A_NF4_MN) {
      g.code2 = src.w->code2;
      g.scale2 = src.w->scale2;
      g.mean = src.w->mean;
    } else if (main_src == A_CHANQ_MN) {
      g.cq_absmax = src.cq_absmax;
    }
    g.epi = EPI_BF16;
    g.out = dX;
    g.o_rs = 1;
    g.o_cs = K;
    g.out_elems = M * K;
    if (main_src == A_NF4_MN || main_src == A_CHANQ_MN) g.cst_elems = N * (K / 64);
    CUtensorMap mo;
    g.stage = stage_map(&mo, dX, K, M, K) ? 1 : 0;
    g.part = part;
    g.counters = cnt;
    if (g_ev_start) cudaEventRecord(g_ev_start, s);
    st = launch_any(L.main, ma, mb, mbx, mo, mt, g, s);
    if (g_ev_stop) cudaEventRecord(g_ev_stop, s);
    if (st != QNF4_OK) return st;
  }
  return QNF4_OK;
}

qnf4_status check_linear_args(int64_t N, int64_t K, int64_t M, int r, bool bwd,
                              std::initializer_list<const void*> ptrs) {
  if (N <= 0 || K <= 0) return fail(QNF4_ERR_SHAPE, "N and K must be positive");
  if (K % 64) return fail(QNF4_ERR_SHAPE, "K must be a multiple of 64 (got %lld)", (long long)K);
  if (bwd && N % 8) return fail(QNF4_ERR_SHAPE, "the backward needs N to be a multiple of 8 (got %lld)", (long long)N);
  if (M < 0) return fail(QNF4_ERR_SHAPE, "M must be >= 0");
  if (M > (int64_t)INT32_MAX) return fail(QNF4_ERR_SHAPE, "M too large");
  if (r < 1 || r > 64) return fail(QNF4_ERR_ARG, "r must be in [1, 64] (got %d)", r);
  for (const void* p : ptrs) {
    if (!p) return fail(QNF4_ERR_ARG, "NULL buffer");
    if (!al16(p)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  }
  return QNF4_OK;
}


// ---------------------------------------------------------------------------
// Workspace for the allocation-free forward (qnf4_qlora_linear_fwd_noalloc). A
// file-scope device array: every GPU that loads the library holds it until exit.
// 32 MiB covers the forward's split-K partial tiles at their largest (one 256-column
// tile slice per CTA slot: 148 x 256 x 128 fp32 on a B200, 19.4 MB), the adapter
// projection's partials and the bf16 (s u) rows (128 bytes per token) up to 65536
// tokens, for every N, K and r <= 64.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on each device, looked up once per device with that
// device current (cudaGetSymbolAddress); later calls read the cached address without
// taking the lock. nullptr and a message on failure.
void* noalloc_scratch_ptr() {
  constexpr int kMaxDev = 64;
  static std::atomic<void*> cache[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) {
    fail(QNF4_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(ge));
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDev) {
    fail(QNF4_ERR_CUDA, "device %d out of range for the built-in scratch (at most %d devices)", dev, kMaxDev);
    return nullptr;
  }
  if (void* p = cache[dev].load(std::memory_order_acquire)) return p;
  std::lock_guard<std::mutex> lk(mu);
  if (void* p = cache[dev].load(std::memory_order_relaxed)) return p;
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) {
    fail(QNF4_ERR_CUDA, "scratch address: %s", cudaGetErrorString(e));
    return nullptr;
  }
  cache[dev].store(p, std::memory_order_release);
  return p;
}
// ---------------------------------------------------------------------------
// Dense linear algebra for the LoftQ initialisation's truncated SVD: cuBLAS (sgemm) and
// cuSOLVER (syevd), loaded at first use by soname (torch's copies when torch has loaded
// them, else the toolkit's), so the library still loads where they are absent.
// ---------------------------------------------------------------------------
struct LinAlgLib {
  bool ok = false;
  decltype(&cublasCreate_v2) blas_create = nullptr;
  decltype(&cublasSetStream_v2) blas_stream = nullptr;
  decltype(&cublasSgemm_v2) sgemm = nullptr;
  decltype(&cusolverDnCreate) sol_create = nullptr;
  decltype(&cusolverDnSetStream) sol_stream = nullptr;
  decltype(&cusolverDnSsyevd_bufferSize) syevd_size = nullptr;
  decltype(&cusolverDnSsyevd) syevd = nullptr;
};

const LinAlgLib& linalg_lib() {
  static const LinAlgLib lib = [] {
    LinAlgLib l;
    auto open = [](std::initializer_list<const char*> names) -> void* {
      for (const char* n : names)
        if (void* h = dlopen(n, RTLD_NOW | RTLD_GLOBAL)) return h;
      return nullptr;
    };
    void* hb = open({"libcublas.so.12", "/usr/local/cuda/lib64/libcublas.so.12", "libcublas.so"});
    void* hs = open({"libcusolver.so.11", "/usr/local/cuda/lib64/libcusolver.so.11", "libcusolver.so"});
    if (!hb || !hs) return l;
    l.blas_create = reinterpret_cast<decltype(l.blas_create)>(dlsym(hb, "cublasCreate_v2"));
    l.blas_stream = reinterpret_cast<decltype(l.blas_stream)>(dlsym(hb, "cublasSetStream_v2"));
    l.sgemm = reinterpret_cast<decltype(l.sgemm)>(dlsym(hb, "cublasSgemm_v2"));
    l.sol_create = reinterpret_cast<decltype(l.sol_create)>(dlsym(hs, "cusolverDnCreate"));
    l.sol_stream = reinterpret_cast<decltype(l.sol_stream)>(dlsym(hs, "cusolverDnSetStream"));
    l.syevd_size = reinterpret_cast<decltype(l.syevd_size)>(dlsym(hs, "cusolverDnSsyevd_bufferSize"));
    l.syevd = reinterpret_cast<decltype(l.syevd)>(dlsym(hs, "cusolverDnSsyevd"));
    l.ok = l.blas_create && l.blas_stream && l.sgemm && l.sol_create && l.sol_stream &&
           l.syevd_size && l.syevd;
    return l;
  }();
  return lib;
}

// One cuBLAS and one cuSOLVER handle per device, kept for the process.
bool linalg_handles(cublasHandle_t* hb, cusolverDnHandle_t* hs) {
  const LinAlgLib& L = linalg_lib();
  if (!L.ok) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return false;
  static std::mutex mu;
  static cublasHandle_t b[64] = {};
  static cusolverDnHandle_t so[64] = {};
  std::lock_guard<std::mutex> lk(mu);
  if (!b[dev] && L.blas_create(&b[dev]) != CUBLAS_STATUS_SUCCESS) return false;
  if (!so[dev] && L.sol_create(&so[dev]) != CUSOLVER_STATUS_SUCCESS) return false;
  *hb = b[dev];
  *hs = so[dev];
  return true;
}

// Floats of syevd workspace for an m x m Gram matrix: the library's own query when a GPU
// and cuSOLVER are at hand, and never below the LAPACK bound 1 + 6m + 2m^2.
size_t loftq_lwork(int64_t m) {
  size_t need = 1 + 6 * static_cast<size_t>(m) + 2 * static_cast<size_t>(m) * static_cast<size_t>(m);
  cublasHandle_t hb;
  cusolverDnHandle_t hs;
  if (linalg_handles(&hb, &hs)) {
    int lw = 0;
    if (linalg_lib().syevd_size(hs, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, static_cast<int>(m),
                                nullptr, static_cast<int>(m), nullptr, &lw) == CUSOLVER_STATUS_SUCCESS)
      need = std::max(need, static_cast<size_t>(lw));
  }
  return need;
}

struct LoftqLayout {
  size_t tgt, q, absmax, dq, gram, eig, p, info, work, total;
  int64_t m;
  size_t lwork;
};

LoftqLayout loftq_layout(int64_t N, int64_t K, int r) {
  LoftqLayout l{};
  l.m = std::min(N, K);
  l.lwork = loftq_lwork(l.m);
  size_t o = 0;
  l.tgt = o;    o = align256(o + static_cast<size_t>(N) * K * 2);
  l.q = o;      o = align256(o + static_cast<size_t>(N) * K * 4);
  l.absmax = o; o = align256(o + static_cast<size_t>(N) * K / 64 * 4);
  l.dq = o;     o = align256(o + qnf4_workspace_size(QNF4_OP_DOUBLE_QUANT, 0, 0, 0, 0));
  l.gram = o;   o = align256(o + static_cast<size_t>(l.m) * l.m * 4);
  l.eig = o;    o = align256(o + static_cast<size_t>(l.m) * 4);
  l.p = o;      o = align256(o + static_cast<size_t>(l.m) * r * 4);
  l.info = o;   o = align256(o + 16);
  l.work = o;   o = align256(o + l.lwork * 4);
  l.total = o;
  return l;
}

}  // namespace
}  // namespace qnf4

using namespace qnf4;

// NVTX range around each ABI call (named after the call), for timeline tools; a
// no-op unless a tool is attached to the process.
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

extern "C" {

qnf4_status qnf4_nf4_codebook(float levels[16], float thresholds[15]) {
  const Nf4Tables& t = nf4_tables();
  if (levels) std::memcpy(levels, t.levels, 16 * sizeof(float));
  if (thresholds) std::memcpy(thresholds, t.thr, 15 * sizeof(float));
  return QNF4_OK;
}

const char* qnf4_last_error(void) { return g_last.c_str(); }

unsigned long long qnf4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }


qnf4_status qnf4_set_timing_events(void* start, void* stop) {
  if ((start == nullptr) != (stop == nullptr)) return fail(QNF4_ERR_ARG, "give both events or neither");
  g_ev_start = static_cast<cudaEvent_t>(start);
  g_ev_stop = static_cast<cudaEvent_t>(stop);
  return QNF4_OK;
}

qnf4_status qnf4_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) return fail(QNF4_ERR_ARG, "timeout must be positive");
  g_wait_ns = ns;
  return QNF4_OK;
}

qnf4_status qnf4_check(void* stream) {
  TraceRange trace_("qnf4_check");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(QNF4_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
  unsigned int flag = 0;
  e = cudaMemcpyFromSymbol(&flag, g_qnf4_err, sizeof(flag));
  if (e != cudaSuccess) return fail(QNF4_ERR_CUDA, "error flag: %s", cudaGetErrorString(e));
  if (flag) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_qnf4_err, &zero, sizeof(zero));
    if (flag == kErrEigensolve) return fail(QNF4_ERR_CUDA, "LoftQ eigensolve failed (cuSOLVER info != 0)");
    if (flag >= kErrBoundsBase)
      return fail(QNF4_ERR_BOUNDS, "a kernel index fell outside its buffer (site %u)", flag - kErrBoundsBase);
    return fail(QNF4_ERR_TIMEOUT, "a kernel wait gave up (site %u)", flag);
  }
  return QNF4_OK;
}

size_t qnf4_workspace_size(int32_t op, int64_t N, int64_t K, int64_t M, int32_t r) {
  switch (op) {
    case QNF4_OP_QUANTIZE: return kQuantMaxGrid * sizeof(double);
    case QNF4_OP_LAYER_STATS: return 2 * kQuantMaxGrid * sizeof(double);
    case QNF4_OP_QUANTIZE_WEIGHT: return 2 * kQuantMaxGrid * sizeof(double);
    case QNF4_OP_QUANTIZE_WEIGHT_GROUP: return 2 * kQMaxJobs * kQuantMaxGrid * sizeof(double);
    case QNF4_OP_LAYER_STATS_GROUP: return 2 * kQMaxJobs * kQuantMaxGrid * sizeof(double);
    case QNF4_OP_DOUBLE_QUANT: return kDqPartials * sizeof(double);
    case QNF4_OP_FWD: {
      const size_t t = plan_linear(A_NF4_K, N, K, M, r, false, num_sms()).total;
      return M <= kDecodeMaxTokens ? std::max(t, decode_ws_bytes(K, M, r)) : t;
    }
    case QNF4_OP_BWD: return plan_linear(A_NF4_MN, N, K, M, r, true, num_sms()).total;
    case QNF4_OP_CHANQ_FWD: return plan_linear(A_CHANQ_K, N, K, M, r, false, num_sms()).total;
    case QNF4_OP_LOFTQ: return loftq_layout(N, K, r).total;
    case QNF4_OP_CHANQ_BWD: {
      const size_t t = plan_linear(A_CHANQ_MN, N, K, M, r, true, num_sms()).total;
      return t + chanq_wide_bytes(N, K);
    }
    default: return 0;
  }
}

qnf4_status qnf4_nf4_quantize(const void* W, int64_t N, int64_t K, int32_t block1, uint8_t* packed,
                              float* absmax, double* sse, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_nf4_quantize");
  if (block1 != 64) return fail(QNF4_ERR_ARG, "block1 must be 64");
  if (N < 0 || K <= 0) return fail(QNF4_ERR_SHAPE, "bad shape");
  if (K % 64) return fail(QNF4_ERR_SHAPE, "K must be a multiple of 64");
  if (!W || !packed || !absmax) return fail(QNF4_ERR_ARG, "NULL buffer");
  if (!al16(W) || !al16(packed) || !al16(absmax) || (sse && !al16(sse)))
    return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (sse && (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_QUANTIZE, N, K, 0, 0)))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nblocks = N * K / 64;
  if (nblocks == 0) {
    if (sse) cudaMemsetAsync(sse, 0, sizeof(double), s);
    return launched("quantize(empty)", 0);
  }
  qnf4_status st = quant_smem_attr();
  if (st != QNF4_OK) return st;
  const int grid = quant_grid(nblocks);
  static thread_local QuantJobs jobs;
  if (!one_quant_job(&jobs, W, nblocks, packed, absmax)) return map_fail();
  const QuantTab tab = make_tab();
  if (sse) {
    launch_pdl(k_nf4_quant<true, true>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs,
               static_cast<double*>(ws), tab, g_wait_ns, 0.f, static_cast<double*>(nullptr),
               static_cast<double*>(nullptr));
    launch_pdl(k_sum_partials, dim3(1), dim3(256), 0, s, static_cast<const double*>(ws), grid, sse);
    return launched("nf4_quantize", 2);
  }
  launch_pdl(k_nf4_quant<true, false>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs,
             static_cast<double*>(nullptr), tab, g_wait_ns, 0.f, static_cast<double*>(nullptr),
             static_cast<double*>(nullptr));
  return launched("nf4_quantize");
}

qnf4_status qnf4_quantize_weight(const void* W, int64_t N, int64_t K, uint8_t* packed, float* absmax,
                                 uint8_t* code2, float* scale2, float* mean, double* sse, void* ws,
                                 size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_quantize_weight");
  if (N <= 0 || K <= 0) return fail(QNF4_ERR_SHAPE, "N and K must be positive");
  if (K % 64) return fail(QNF4_ERR_SHAPE, "K must be a multiple of 64");
  if (!W || !packed || !absmax || !code2 || !scale2 || !mean) return fail(QNF4_ERR_ARG, "NULL buffer");
  for (const void* p : {W, static_cast<const void*>(packed), static_cast<const void*>(absmax),
                        static_cast<const void*>(code2), static_cast<const void*>(scale2),
                        static_cast<const void*>(mean)})
    if (!al16(p)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (sse && !al16(sse)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_QUANTIZE_WEIGHT, N, K, 0, 0))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  qnf4_status st = quant_smem_attr();
  if (st != QNF4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nblocks = N * K / 64;
  const int grid = quant_grid(nblocks);
  static thread_local QuantJobs jobs;
  if (!one_quant_job(&jobs, W, nblocks, packed, absmax)) return map_fail();
  double* asum = static_cast<double*>(ws);
  double* ssep = asum + kQuantMaxGrid;
  const QuantTab tab = make_tab();
  if (sse) {
    launch_pdl(k_nf4_quant<true, true>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs, ssep, tab,
               g_wait_ns, 0.f, static_cast<double*>(nullptr), asum);
  } else {
    launch_pdl(k_nf4_quant<true, false>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs,
               static_cast<double*>(nullptr), tab, g_wait_ns, 0.f, static_cast<double*>(nullptr), asum);
  }
  static thread_local DqJobs dq;
  const int egrid = one_dq_job(&dq, absmax, nblocks, asum, grid, nblocks, code2, scale2, mean,
                               sse ? ssep : nullptr, grid, sse);
  launch_pdl(k_dq_encode, dim3(egrid), dim3(256), 0, s, dq);
  return launched("quantize_weight", 2);
}

qnf4_status qnf4_quantize_weight_group(int32_t n, const void* const* W, const int64_t* N,
                                       const int64_t* K, uint8_t* const* packed, float* const* absmax,
                                       uint8_t* const* code2, float* const* scale2, float* const* mean,
                                       double* const* sse, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_quantize_weight_group");
  if (n < 1 || n > kQMaxJobs) return fail(QNF4_ERR_ARG, "n must be in [1, %d] (got %d)", kQMaxJobs, n);
  if (!W || !N || !K || !packed || !absmax || !code2 || !scale2 || !mean) return fail(QNF4_ERR_ARG, "NULL array");
  for (int l = 0; l < n; ++l) {
    if (N[l] <= 0 || K[l] <= 0) return fail(QNF4_ERR_SHAPE, "weight %d: N and K must be positive", l);
    if (K[l] % 64) return fail(QNF4_ERR_SHAPE, "weight %d: K must be a multiple of 64", l);
    if (!W[l] || !packed[l] || !absmax[l] || !code2[l] || !scale2[l] || !mean[l] || (sse && !sse[l]))
      return fail(QNF4_ERR_ARG, "weight %d: NULL buffer", l);
    for (const void* p : {W[l], static_cast<const void*>(packed[l]), static_cast<const void*>(absmax[l]),
                          static_cast<const void*>(code2[l]), static_cast<const void*>(scale2[l]),
                          static_cast<const void*>(mean[l]), static_cast<const void*>(sse ? sse[l] : nullptr)})
      if (p && !al16(p)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  }
  if (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_QUANTIZE_WEIGHT_GROUP, 0, 0, 0, 0))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  qnf4_status st = quant_smem_attr();
  if (st != QNF4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local QuantJobs jobs;
  static thread_local DqJobs dq;
  std::memset(&jobs, 0, sizeof(jobs));
  std::memset(&dq, 0, sizeof(dq));
  jobs.n = dq.n = n;
  jobs.chunk0[0] = dq.b2_0[0] = 0;
  double* asum = static_cast<double*>(ws);
  double* ssep = asum + kQMaxJobs * kQuantMaxGrid;
  for (int l = 0; l < n; ++l) {
    const int64_t nb = N[l] * K[l] / 64;
    jobs.nblocks[l] = nb;
    jobs.chunk0[l + 1] = jobs.chunk0[l] + (nb + kQChunkBlocks - 1) / kQChunkBlocks;
    jobs.packed[l] = reinterpret_cast<uint32_t*>(packed[l]);
    jobs.absmax[l] = absmax[l];
    if (!quant_map(&jobs.map[l], W[l], nb)) return map_fail();
    dq.c[l] = absmax[l];
    dq.nb1[l] = nb;
    dq.count[l] = nb;
    dq.part[l] = asum + l * kQuantMaxGrid;
    dq.code2[l] = code2[l];
    dq.scale2[l] = scale2[l];
    dq.mean[l] = mean[l];
    dq.sse_part[l] = ssep + l * kQuantMaxGrid;
    dq.sse_out[l] = sse ? sse[l] : nullptr;
    dq.b2_0[l + 1] = dq.b2_0[l] + (nb + 255) / 256;
  }
  const int grid = quant_grid_chunks(jobs.chunk0[n]);
  dq.npart = dq.nsse = grid;
  const QuantTab tab = make_tab();
  if (sse) {
    launch_pdl(k_nf4_quant<true, true>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs, ssep, tab,
               g_wait_ns, 0.f, static_cast<double*>(nullptr), asum);
  } else {
    launch_pdl(k_nf4_quant<true, false>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs,
               static_cast<double*>(nullptr), tab, g_wait_ns, 0.f, static_cast<double*>(nullptr), asum);
  }
  const int egrid = std::max(dq_grid(&dq, dq.b2_0[n]), n);  // CTA l < n folds weight l's SSE
  launch_pdl(k_dq_encode, dim3(egrid), dim3(256), 0, s, dq);
  return launched("quantize_weight_group", 2);
}

qnf4_status qnf4_nf4_layer_stats_group(int32_t n, const void* const* W, const int64_t* N,
                                       const int64_t* K, float tau, double* const* sse,
                                       double* const* below, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_nf4_layer_stats_group");
  if (n < 1 || n > kQMaxJobs) return fail(QNF4_ERR_ARG, "n must be in [1, %d] (got %d)", kQMaxJobs, n);
  if (!W || !N || !K || !sse) return fail(QNF4_ERR_ARG, "NULL array");
  if (below && (!(tau >= 0.f) || std::isinf(tau))) return fail(QNF4_ERR_ARG, "tau must be finite and >= 0");
  for (int l = 0; l < n; ++l) {
    if (N[l] <= 0 || K[l] <= 0) return fail(QNF4_ERR_SHAPE, "weight %d: N and K must be positive", l);
    if (K[l] % 64) return fail(QNF4_ERR_SHAPE, "weight %d: K must be a multiple of 64", l);
    if (!W[l] || !sse[l] || (below && !below[l])) return fail(QNF4_ERR_ARG, "weight %d: NULL buffer", l);
    if (!al16(W[l]) || !al16(sse[l]) || (below && !al16(below[l])))
      return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  }
  if (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_LAYER_STATS_GROUP, 0, 0, 0, 0))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  qnf4_status st = quant_smem_attr();
  if (st != QNF4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local QuantJobs jobs;
  std::memset(&jobs, 0, sizeof(jobs));
  jobs.n = n;
  SumJobs sj;
  std::memset(&sj, 0, sizeof(sj));
  for (int l = 0; l < n; ++l) {
    const int64_t nb = N[l] * K[l] / 64;
    jobs.nblocks[l] = nb;
    jobs.chunk0[l + 1] = jobs.chunk0[l] + (nb + kQChunkBlocks - 1) / kQChunkBlocks;
    if (!quant_map(&jobs.map[l], W[l], nb)) return map_fail();
    sj.out[l] = sse[l];
  }
  const int grid = quant_grid_chunks(jobs.chunk0[n]);
  double* part = static_cast<double*>(ws);  // SSE partials, then the counts', per job
  const QuantTab tab = make_tab();
  if (below) {
    launch_pdl(k_nf4_quant<false, true, true>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs, part, tab,
               g_wait_ns, tau, part + kQMaxJobs * kQuantMaxGrid, static_cast<double*>(nullptr));
  } else {
    launch_pdl(k_nf4_quant<false, true>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs, part, tab,
               g_wait_ns, 0.f, static_cast<double*>(nullptr), static_cast<double*>(nullptr));
  }
  launch_pdl(k_sum_partials_jobs, dim3(n), dim3(256), 0, s, static_cast<const double*>(part), grid, sj);
  if (below) {
    SumJobs sj2;
    std::memset(&sj2, 0, sizeof(sj2));
    for (int l = 0; l < n; ++l) sj2.out[l] = below[l];
    launch_pdl(k_sum_partials_jobs, dim3(n), dim3(256), 0, s,
               static_cast<const double*>(part + kQMaxJobs * kQuantMaxGrid), grid, sj2);
  }
  return launched("nf4_layer_stats_group", below ? 3 : 2);
}

qnf4_status qnf4_nf4_recon_error(const void* W, int64_t N, int64_t K, int32_t block1, double* sse,
                                 void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_nf4_recon_error");
  if (block1 != 64) return fail(QNF4_ERR_ARG, "block1 must be 64");
  if (N < 0 || K <= 0) return fail(QNF4_ERR_SHAPE, "bad shape");
  if (K % 64) return fail(QNF4_ERR_SHAPE, "K must be a multiple of 64");
  if (!W || !sse) return fail(QNF4_ERR_ARG, "NULL buffer");
  if (!al16(W) || !al16(sse)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_QUANTIZE, N, K, 0, 0))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nblocks = N * K / 64;
  if (nblocks == 0) {
    cudaMemsetAsync(sse, 0, sizeof(double), s);
    return launched("recon_error(empty)", 0);
  }
  qnf4_status st = quant_smem_attr();
  if (st != QNF4_OK) return st;
  const int grid = quant_grid(nblocks);
  static thread_local QuantJobs jobs;
  if (!one_quant_job(&jobs, W, nblocks, nullptr, nullptr)) return map_fail();
  launch_pdl(k_nf4_quant<false, true>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs,
             static_cast<double*>(ws), make_tab(), g_wait_ns, 0.f, static_cast<double*>(nullptr),
             static_cast<double*>(nullptr));
  launch_pdl(k_sum_partials, dim3(1), dim3(256), 0, s, static_cast<const double*>(ws), grid, sse);
  return launched("nf4_recon_error", 2);
}

qnf4_status qnf4_nf4_layer_stats(const void* W, int64_t N, int64_t K, float tau, double* sse,
                                 double* below, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_nf4_layer_stats");
  if (N < 0 || K <= 0) return fail(QNF4_ERR_SHAPE, "bad shape");
  if (K % 64) return fail(QNF4_ERR_SHAPE, "K must be a multiple of 64");
  if (!W || !sse || !below) return fail(QNF4_ERR_ARG, "NULL buffer");
  if (!al16(W) || !al16(sse) || !al16(below)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (!(tau >= 0.f) || std::isinf(tau)) return fail(QNF4_ERR_ARG, "tau must be finite and >= 0");
  if (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_LAYER_STATS, N, K, 0, 0))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nblocks = N * K / 64;
  if (nblocks == 0) {
    cudaMemsetAsync(sse, 0, sizeof(double), s);
    cudaMemsetAsync(below, 0, sizeof(double), s);
    return launched("layer_stats(empty)", 0);
  }
  qnf4_status st = quant_smem_attr();
  if (st != QNF4_OK) return st;
  const int grid = quant_grid(nblocks);
  static thread_local QuantJobs jobs;
  if (!one_quant_job(&jobs, W, nblocks, nullptr, nullptr)) return map_fail();
  double* part = static_cast<double*>(ws);
  launch_pdl(k_nf4_quant<false, true, true>, dim3(grid), dim3(kQThreads), kQSmem, s, jobs, part,
             make_tab(), g_wait_ns, tau, part + kQuantMaxGrid, static_cast<double*>(nullptr));
  launch_pdl(k_sum_partials, dim3(1), dim3(256), 0, s, part, grid, sse);
  launch_pdl(k_sum_partials, dim3(1), dim3(256), 0, s, part + kQuantMaxGrid, grid, below);
  return launched("nf4_layer_stats", 3);
}

qnf4_status qnf4_double_quant(const float* absmax, int64_t nb1, int32_t block2, uint8_t* code2,
                              float* scale2, float* mean, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_double_quant");
  if (block2 != 256) return fail(QNF4_ERR_ARG, "block2 must be 256");
  if (nb1 <= 0) return fail(QNF4_ERR_SHAPE, "nb1 must be positive");
  if (!absmax || !code2 || !scale2 || !mean) return fail(QNF4_ERR_ARG, "NULL buffer");
  if (!al16(absmax) || !al16(code2) || !al16(scale2) || !al16(mean))
    return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_DOUBLE_QUANT, 0, 0, 0, 0))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* part = static_cast<double*>(ws);
  k_dq_partial<<<kDqPartials, 256, 0, s>>>(absmax, nb1, part);
  static thread_local DqJobs dq;
  const int grid = one_dq_job(&dq, absmax, nb1, part, kDqPartials, nb1, code2, scale2, mean, nullptr, 0, nullptr);
  launch_pdl(k_dq_encode, dim3(grid), dim3(256), 0, s, dq);
  return launched("double_quant", 2);
}

qnf4_status qnf4_dq_sum(const float* absmax, int64_t nb1, double* sum, void* ws, size_t ws_bytes,
                        void* stream) {
  TraceRange trace_("qnf4_dq_sum");
  if (nb1 <= 0) return fail(QNF4_ERR_SHAPE, "nb1 must be positive");
  if (!absmax || !sum) return fail(QNF4_ERR_ARG, "NULL buffer");
  if (!al16(absmax) || !al16(sum)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (!ws || ws_bytes < qnf4_workspace_size(QNF4_OP_DOUBLE_QUANT, 0, 0, 0, 0))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* part = static_cast<double*>(ws);
  k_dq_partial<<<kDqPartials, 256, 0, s>>>(absmax, nb1, part);
  launch_pdl(k_sum_partials, dim3(1), dim3(256), 0, s, part, kDqPartials, sum);
  return launched("dq_sum", 2);
}

qnf4_status qnf4_double_quant_shard(const float* absmax, int64_t nb1, int32_t block2,
                                    const double* total_sum, int64_t total_count, uint8_t* code2,
                                    float* scale2, float* mean, void* stream) {
  TraceRange trace_("qnf4_double_quant_shard");
  if (block2 != 256) return fail(QNF4_ERR_ARG, "block2 must be 256");
  if (nb1 <= 0) return fail(QNF4_ERR_SHAPE, "nb1 must be positive");
  if (total_count < nb1) return fail(QNF4_ERR_SHAPE, "total_count must be >= nb1");
  if (!absmax || !total_sum || !code2 || !scale2 || !mean) return fail(QNF4_ERR_ARG, "NULL buffer");
  if (!al16(absmax) || !al16(total_sum) || !al16(code2) || !al16(scale2) || !al16(mean))
    return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local DqJobs dq;
  const int grid = one_dq_job(&dq, absmax, nb1, total_sum, 1, total_count, code2, scale2, mean, nullptr, 0, nullptr);
  launch_pdl(k_dq_encode, dim3(grid), dim3(256), 0, s, dq);
  return launched("dq_encode_shard");
}

qnf4_status qnf4_dequant(const qnf4_weight* w, void* out, int32_t out_dtype, void* stream) {
  TraceRange trace_("qnf4_dequant");
  qnf4_status st = check_weight(w);
  if (st != QNF4_OK) return st;
  if (!out) return fail(QNF4_ERR_ARG, "NULL output");
  if (!al16(out)) return fail(QNF4_ERR_ALIGN, "output must be 16-byte aligned");
  if (out_dtype != QNF4_OUT_F32 && out_dtype != QNF4_OUT_BF16)
    return fail(QNF4_ERR_ARG, "out_dtype must be QNF4_OUT_F32 or QNF4_OUT_BF16");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n8 = w->N * w->K / 8;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, num_sms() * 8)));
  const QuantTab tab = make_tab();
  const uint32_t* p = reinterpret_cast<const uint32_t*>(w->packed);
  if (out_dtype == QNF4_OUT_BF16)
    k_dequant<true><<<grid, 256, 0, s>>>(p, w->code2, w->scale2, w->mean, n8, out, tab);
  else
    k_dequant<false><<<grid, 256, 0, s>>>(p, w->code2, w->scale2, w->mean, n8, out, tab);
  return launched("dequant");
}

qnf4_status qnf4_rank_topk(const double* sse, const int64_t* n_params, int32_t n_layers, int32_t k,
                           int32_t* out) {
  if (!sse || !n_params || (!out && k > 0)) return fail(QNF4_ERR_ARG, "NULL host buffer");
  if (n_layers < 0 || k < 0 || k > n_layers) return fail(QNF4_ERR_ARG, "need 0 <= k <= n_layers");
  std::vector<int32_t> idx(n_layers);
  for (int32_t i = 0; i < n_layers; ++i) {
    if (n_params[i] <= 0) return fail(QNF4_ERR_ARG, "n_params must be positive");
    idx[i] = i;
  }
  // epsilon_i = sse_i / n_i, descending; ties to the lower index (stable)
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
    return sse[a] / static_cast<double>(n_params[a]) > sse[b] / static_cast<double>(n_params[b]);
  });
  for (int32_t i = 0; i < k; ++i) out[i] = idx[i];
  return QNF4_OK;
}

qnf4_status qnf4_chanq_quantize(const void* W, int64_t N, int64_t K, const uint8_t* bits,
                                const float* thr, const int64_t* thr_off, uint8_t* packed,
                                const int64_t* row_off, float* absmax, void* stream) {
  TraceRange trace_("qnf4_chanq_quantize");
  if (N < 0 || K <= 0) return fail(QNF4_ERR_SHAPE, "bad shape");
  if (K % 64) return fail(QNF4_ERR_SHAPE, "K must be a multiple of 64");
  if (!W || !bits || !thr || !thr_off || !packed || !row_off || !absmax)
    return fail(QNF4_ERR_ARG, "NULL buffer");
  if (!al16(W) || !al16(bits) || !al16(thr) || !al16(thr_off) || !al16(packed) || !al16(row_off) ||
      !al16(absmax))
    return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  if (N == 0) return QNF4_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((N + 7) / 8, num_sms() * 8)));
  k_chanq_quant<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(W), N, K, bits, thr, thr_off,
                                     packed, row_off, absmax);
  return launched("chanq_quantize");
}

qnf4_status qnf4_qlora_linear_fwd(const qnf4_weight* w, const void* x, int64_t M, const void* A,
                                  const void* B, int32_t r, float scale, void* h, void* ws,
                                  size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_qlora_linear_fwd");
  qnf4_status st = check_weight(w);
  if (st != QNF4_OK) return st;
  st = check_linear_args(w->N, w->K, M, r, false, {x, A, B, h});
  if (st != QNF4_OK) return st;
  if (M == 0) return QNF4_OK;
  if (M <= kDecodeMaxTokens)
    return decode_fwd(w, x, M, A, B, r, scale, h, ws, ws_bytes, static_cast<cudaStream_t>(stream));
  BaseSrc src;
  src.kind = A_NF4_K;
  src.w = w;
  src.N = w->N;
  src.K = w->K;
  return linear_fwd(src, x, M, A, B, r, scale, h, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

qnf4_status qnf4_qlora_linear_fwd_group(int32_t n, const qnf4_weight* w, const void* const* x,
                                        int64_t M, const void* const* A, const void* const* B,
                                        int32_t r, float scale, void* const* h, void* ws,
                                        size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_qlora_linear_fwd_group");
  if (n < 1 || n > kDecMaxGroup) return fail(QNF4_ERR_ARG, "n must be in [1, %d] (got %d)", kDecMaxGroup, n);
  if (!w || !x || !A || !B || !h) return fail(QNF4_ERR_ARG, "NULL array");
  if (M < 1 || M > kDecodeMaxTokens)
    return fail(QNF4_ERR_SHAPE, "the grouped forward takes 1 to %lld tokens (got %lld)",
                static_cast<long long>(kDecodeMaxTokens), static_cast<long long>(M));
  size_t need = 0;
  for (int l = 0; l < n; ++l) {
    qnf4_status st = check_weight(&w[l]);
    if (st != QNF4_OK) return st;
    st = check_linear_args(w[l].N, w[l].K, M, r, false, {x[l], A[l], B[l], h[l]});
    if (st != QNF4_OK) return st;
    need += decode_ws_bytes(w[l].K, M, r);
  }
  if (!ws || ws_bytes < need) return fail(QNF4_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, need);
  return decode_group(n, w, x, M, A, B, r, scale, h, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

qnf4_status qnf4_qlora_linear_fwd_noalloc(const qnf4_weight* w, const void* x, int64_t M,
                                          const void* A, const void* B, int32_t r, float scale,
                                          void* h, void* stream) {
  TraceRange trace_("qnf4_qlora_linear_fwd_noalloc");
  qnf4_status st = check_weight(w);
  if (st != QNF4_OK) return st;
  st = check_linear_args(w->N, w->K, M, r, false, {x, A, B, h});
  if (st != QNF4_OK) return st;
  if (M == 0) return QNF4_OK;
  const size_t need = qnf4_workspace_size(QNF4_OP_FWD, w->N, w->K, M, r);
  if (need > kNoAllocScratchBytes)
    return fail(QNF4_ERR_WORKSPACE,
                "this shape needs %zu bytes of workspace; the built-in scratch holds %zu "
                "(use qnf4_qlora_linear_fwd with a caller-provided workspace)",
                need, kNoAllocScratchBytes);
  void* ws = noalloc_scratch_ptr();
  if (!ws) return QNF4_ERR_CUDA;
  return qnf4_qlora_linear_fwd(w, x, M, A, B, r, scale, h, ws, kNoAllocScratchBytes, stream);
}

qnf4_status qnf4_qlora_linear_bwd(const qnf4_weight* w, const void* x, const void* dY, int64_t M,
                                  const void* A, const void* B, int32_t r, float scale, void* dX,
                                  float* dA, float* dB, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_qlora_linear_bwd");
  qnf4_status st = check_weight(w);
  if (st != QNF4_OK) return st;
  st = check_linear_args(w->N, w->K, M, r, true, {x, dY, A, B, dX, dA, dB});
  if (st != QNF4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    cudaMemsetAsync(dA, 0, sizeof(float) * r * w->K, s);
    cudaMemsetAsync(dB, 0, sizeof(float) * r * w->N, s);
    return launched("bwd(M=0)", 0);
  }
  BaseSrc src;
  src.kind = A_NF4_K;
  src.w = w;
  src.N = w->N;
  src.K = w->K;
  return linear_bwd(src, x, dY, M, A, B, r, scale, dX, dA, dB, ws, ws_bytes, s);
}

qnf4_status qnf4_dense_linear_fwd(const void* W, int64_t N, int64_t K, const void* x, int64_t M,
                                  const void* A, const void* B, int32_t r, float scale, void* h,
                                  void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_dense_linear_fwd");
  qnf4_status st = check_linear_args(N, K, M, r, false, {W, x, A, B, h});
  if (st != QNF4_OK) return st;
  if (M == 0) return QNF4_OK;
  BaseSrc src;
  src.kind = A_DENSE_K;
  src.Wd = W;
  src.N = N;
  src.K = K;
  return linear_fwd(src, x, M, A, B, r, scale, h, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

qnf4_status qnf4_dense_linear_bwd(const void* W, int64_t N, int64_t K, const void* x, const void* dY,
                                  int64_t M, const void* A, const void* B, int32_t r, float scale,
                                  void* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                                  void* stream) {
  TraceRange trace_("qnf4_dense_linear_bwd");
  qnf4_status st = check_linear_args(N, K, M, r, true, {W, x, dY, A, B, dX, dA, dB});
  if (st != QNF4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    cudaMemsetAsync(dA, 0, sizeof(float) * r * K, s);
    cudaMemsetAsync(dB, 0, sizeof(float) * r * N, s);
    return launched("bwd(M=0)", 0);
  }
  BaseSrc src;
  src.kind = A_DENSE_K;
  src.Wd = W;
  src.N = N;
  src.K = K;
  return linear_bwd(src, x, dY, M, A, B, r, scale, dX, dA, dB, ws, ws_bytes, s);
}

qnf4_status qnf4_chanq_linear_fwd(const uint8_t* packed, const int64_t* row_off, const uint8_t* bits,
                                  const float* map, const int64_t* map_off, const float* absmax,
                                  int64_t N, int64_t K, const void* x, int64_t M, const void* A,
                                  const void* B, int32_t r, float scale, void* h, void* ws,
                                  size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_chanq_linear_fwd");
  qnf4_status st = check_linear_args(N, K, M, r, false, {packed, row_off, bits, map, map_off, absmax, x, A, B, h});
  if (st != QNF4_OK) return st;
  if (M == 0) return QNF4_OK;
  BaseSrc src;
  src.kind = A_CHANQ_K;
  src.cq_packed = packed;
  src.cq_row_off = row_off;
  src.cq_bits = bits;
  src.cq_map = map;
  src.cq_map_off = map_off;
  src.cq_absmax = absmax;
  src.N = N;
  src.K = K;
  return linear_fwd(src, x, M, A, B, r, scale, h, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

qnf4_status qnf4_chanq_learn(const void* W_bf16, int64_t N, int64_t K, int32_t bits,
                             const float* thr0, int32_t iters, float* map, float* thr,
                             double* err, int32_t* iters_done, void* stream) {
  TraceRange trace_("qnf4_chanq_learn");
  for (const void* p : {W_bf16, static_cast<const void*>(thr0), static_cast<const void*>(map),
                        static_cast<const void*>(thr), static_cast<const void*>(err)}) {
    if (!p) return fail(QNF4_ERR_ARG, "NULL buffer");
    if (!al16(p)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  }
  if (bits != 1 && bits != 2 && bits != 4) return fail(QNF4_ERR_ARG, "bits must be 1, 2 or 4 (got %d)", bits);
  if (iters < 1) return fail(QNF4_ERR_ARG, "iters must be >= 1");
  if (N < 0 || K <= 0 || K % 64) return fail(QNF4_ERR_SHAPE, "K must be a positive multiple of 64");
  if (K > 32768) return fail(QNF4_ERR_SHAPE, "K at most 32768 (the row lives in shared memory)");
  if (N == 0) return QNF4_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t smem = static_cast<size_t>(K) * 4 + static_cast<size_t>(K / 64) * 4;
  const int grid = static_cast<int>(std::min<int64_t>(N, static_cast<int64_t>(num_sms()) * 4));
  auto go = [&](auto kern) -> qnf4_status {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
      return fail(QNF4_ERR_CUDA, "shared memory attribute refused");
    kern<<<grid, kLearnThreads, smem, s>>>(static_cast<const uint16_t*>(W_bf16), N, K, thr0, iters, map,
                                           thr, err, iters_done);
    return launched("chanq_learn");
  };
  if (bits == 1) return go(k_chanq_learn<2>);
  if (bits == 2) return go(k_chanq_learn<4>);
  return go(k_chanq_learn<16>);
}

qnf4_status qnf4_loftq_nf4(const void* W_bf16, int64_t N, int64_t K, int32_t r, int32_t steps,
                           uint8_t* packed, uint8_t* code2, float* scale2, float* mean, float* A,
                           float* B, double* errs, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_loftq_nf4");
  for (const void* p : {W_bf16, static_cast<const void*>(packed), static_cast<const void*>(code2),
                        static_cast<const void*>(scale2), static_cast<const void*>(mean),
                        static_cast<const void*>(A), static_cast<const void*>(B),
                        static_cast<const void*>(errs)}) {
    if (!p) return fail(QNF4_ERR_ARG, "NULL buffer");
    if (!al16(p)) return fail(QNF4_ERR_ALIGN, "buffers must be 16-byte aligned");
  }
  if (N <= 0 || K <= 0 || K % 64) return fail(QNF4_ERR_SHAPE, "N > 0 and K a positive multiple of 64");
  if (r < 1 || r > std::min(N, K)) return fail(QNF4_ERR_ARG, "r must be in [1, min(N, K)]");
  if (steps < 1) return fail(QNF4_ERR_ARG, "steps must be >= 1");
  if (std::min(N, K) > 16384) return fail(QNF4_ERR_SHAPE, "min(N, K) at most 16384 (the Gram matrix)");
  cublasHandle_t hb;
  cusolverDnHandle_t hs;
  if (!linalg_handles(&hb, &hs)) return fail(QNF4_ERR_CUDA, "cuBLAS / cuSOLVER unavailable");
  const LoftqLayout l = loftq_layout(N, K, r);
  if (!ws || ws_bytes < l.total) return fail(QNF4_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, l.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const LinAlgLib& L = linalg_lib();
  if (L.blas_stream(hb, s) != CUBLAS_STATUS_SUCCESS || L.sol_stream(hs, s) != CUSOLVER_STATUS_SUCCESS)
    return fail(QNF4_ERR_CUDA, "cuBLAS / cuSOLVER stream");
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  uint16_t* tgt = reinterpret_cast<uint16_t*>(w8 + l.tgt);
  float* Q = reinterpret_cast<float*>(w8 + l.q);
  float* absmax = reinterpret_cast<float*>(w8 + l.absmax);
  float* G = reinterpret_cast<float*>(w8 + l.gram);
  float* eig = reinterpret_cast<float*>(w8 + l.eig);
  float* P = reinterpret_cast<float*>(w8 + l.p);
  int* info = reinterpret_cast<int*>(w8 + l.info);
  float* work = reinterpret_cast<float*>(w8 + l.work);
  const int64_t m = l.m;
  const bool gram_k = N >= K;  // Gram R^T R (K x K) when N >= K, else R R^T (N x N)
  cudaMemsetAsync(A, 0, sizeof(float) * r * K, s);
  cudaMemsetAsync(B, 0, sizeof(float) * N * r, s);
  qnf4_weight wq{N, K, 64, 256, packed, code2, scale2, mean};
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((N * K + 255) / 256, num_sms() * 8)));
  const float one = 1.f, zero = 0.f;
  for (int t = 0; t < steps; ++t) {
    k_loftq_target<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(W_bf16), B, A, N, K, r, tgt);
    qnf4_status st = launched("loftq_target");
    if (st != QNF4_OK) return st;
    st = qnf4_nf4_quantize(tgt, N, K, 64, packed, absmax, nullptr, nullptr, 0, stream);
    if (st != QNF4_OK) return st;
    st = qnf4_double_quant(absmax, N * K / 64, 256, code2, scale2, mean, w8 + l.dq,
                           qnf4_workspace_size(QNF4_OP_DOUBLE_QUANT, 0, 0, 0, 0), stream);
    if (st != QNF4_OK) return st;
    st = qnf4_dequant(&wq, Q, QNF4_OUT_F32, stream);
    if (st != QNF4_OK) return st;
    k_loftq_residual<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(W_bf16), Q, N * K);
    st = launched("loftq_residual");
    if (st != QNF4_OK) return st;
    // R row-major [N, K] is column-major K x N with leading dimension K
    const cublasStatus_t g1 =
        gram_k ? L.sgemm(hb, CUBLAS_OP_N, CUBLAS_OP_T, static_cast<int>(K), static_cast<int>(K),
                         static_cast<int>(N), &one, Q, static_cast<int>(K), Q, static_cast<int>(K), &zero, G,
                         static_cast<int>(K))
               : L.sgemm(hb, CUBLAS_OP_T, CUBLAS_OP_N, static_cast<int>(N), static_cast<int>(N),
                         static_cast<int>(K), &one, Q, static_cast<int>(K), Q, static_cast<int>(K), &zero, G,
                         static_cast<int>(N));
    if (g1 != CUBLAS_STATUS_SUCCESS) return fail(QNF4_ERR_CUDA, "cuBLAS sgemm (Gram) failed");
    if (L.syevd(hs, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, static_cast<int>(m), G,
                static_cast<int>(m), eig, work, static_cast<int>(l.lwork), info) != CUSOLVER_STATUS_SUCCESS)
      return fail(QNF4_ERR_CUDA, "cuSOLVER syevd failed");
    const int fg = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((m * r + 255) / 256, num_sms() * 4)));
    // top-r eigenvectors: Gram on the K side gives V (A = rho V^T, B = R V / rho), on the
    // N side U (B = rho U, A^T = R^T U / rho)
    k_loftq_factor<<<fg, 256, 0, s>>>(G, eig, m, r, P, gram_k ? A : B, gram_k ? 0 : 1);
    st = launched("loftq_factor");
    if (st != QNF4_OK) return st;
    const cublasStatus_t g2 =
        gram_k ? L.sgemm(hb, CUBLAS_OP_T, CUBLAS_OP_N, r, static_cast<int>(N), static_cast<int>(K), &one, P,
                         static_cast<int>(K), Q, static_cast<int>(K), &zero, B, r)
               : L.sgemm(hb, CUBLAS_OP_N, CUBLAS_OP_N, static_cast<int>(K), r, static_cast<int>(N), &one, Q,
                         static_cast<int>(K), P, static_cast<int>(N), &zero, A, static_cast<int>(K));
    if (g2 != CUBLAS_STATUS_SUCCESS) return fail(QNF4_ERR_CUDA, "cuBLAS sgemm (factor) failed");
    k_loftq_err<<<1, 256, 0, s>>>(eig, m, r, info, errs + t);
    st = launched("loftq_err");
    if (st != QNF4_OK) return st;
  }
  return QNF4_OK;
}

qnf4_status qnf4_chanq_linear_bwd(const uint8_t* packed, const int64_t* row_off, const uint8_t* bits,
                                  const float* map, const int64_t* map_off, const float* absmax,
                                  int64_t N, int64_t K, const void* x, const void* dY, int64_t M,
                                  const void* A, const void* B, int32_t r, float scale, void* dX,
                                  float* dA, float* dB, void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("qnf4_chanq_linear_bwd");
  qnf4_status st = check_linear_args(N, K, M, r, true,
                                     {packed, row_off, bits, map, map_off, absmax, x, dY, A, B, dX, dA, dB});
  if (st != QNF4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    cudaMemsetAsync(dA, 0, sizeof(float) * r * K, s);
    cudaMemsetAsync(dB, 0, sizeof(float) * r * N, s);
    return launched("bwd(M=0)", 0);
  }
  const size_t own = plan_linear(A_CHANQ_MN, N, K, M, r, true, num_sms()).total;
  if (!ws || ws_bytes < own + chanq_wide_bytes(N, K))
    return fail(QNF4_ERR_WORKSPACE, "workspace too small (%zu < %zu)", ws_bytes, own + chanq_wide_bytes(N, K));
  BaseSrc src;
  src.kind = A_CHANQ_K;
  src.cq_packed = packed;
  src.cq_row_off = row_off;
  src.cq_bits = bits;
  src.cq_map = map;
  src.cq_map_off = map_off;
  src.cq_absmax = absmax;
  src.cq_wide = static_cast<uint8_t*>(ws) + own;
  src.cq_tab = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + own +
                                        align256(static_cast<size_t>(N) * static_cast<size_t>(K / 2)));
  src.N = N;
  src.K = K;
  {
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((N + 7) / 8, num_sms() * 8)));
    k_chanq_widen<<<grid, 256, 0, s>>>(packed, row_off, bits, map, map_off, N, K, src.cq_wide, src.cq_tab);
    st = launched("chanq_widen");
    if (st != QNF4_OK) return st;
  }
  return linear_bwd(src, x, dY, M, A, B, r, scale, dX, dA, dB, ws, own, s);
}

}  // extern "C"
