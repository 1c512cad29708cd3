// One tcgen05 (5th-generation tensor core) GEMM skeleton for every contraction of
// the QLoRA linear layer, with the A operand produced in one of five ways.
//
//   D[rows, cols] = sum_c Aop[row, c] * Bop[col, c]   (+ one extra "LoRA" chunk)
//
// The M side of the MMA ("rows", 128 per CTA) is the A operand; the N side ("cols",
// tn per CTA, 16..256) is the B operand, always bf16 and K-major, loaded by TMA with
// the 128-byte swizzle. The contraction runs in steps of 64.
//
// A operand sources:
//   A_NF4_K    packed NF4 weight, rows = output features, contraction = input features
//              (forward h = x W^T). TMA brings the packed bytes; converter warps
//              dequantize each 64-element block with its two-level constant and
//              write bf16 into a K-major SW128 tile.
//   A_NF4_MN   packed NF4 weight read transposed: rows = input features, contraction
//              = output features (backward dX = dY W). Same converter, MN-major tile.
//   A_DENSE_K  bf16 matrix by TMA, K-major (dense layers, x for u = x A^T, dY for v).
//   A_DENSE_MN bf16 matrix by TMA, MN-major (dense dX, x^T for dA, dY^T for dB).
//   A_CHANQ_K  per-output-channel 1/2/4-bit codes with per-row mapping tables,
//              widened to the 4-bit layout and looked up like NF4 (A in tensor memory).
//
// The extra chunk adds sum_j Aext[row, j] * Bext[col, j] over j < r into the same
// TMEM accumulator: the rank-r adapter term of "QLoRA: Efficient Finetuning of
// Quantized LLMs" (Heng's Blog, opening formula h = dequant(W0) x + (alpha/r) B A x).
//
// Roles (64 + 128 NSET threads): warp 0 issues TMA, warp 1 allocates TMEM and one
// lane issues tcgen05.mma, and NSET sets of four "converter" warps dequantize (set h
// takes the steps i with i % NSET == h, one 64-element NF4 block per thread and
// step) and then run the epilogue (tcgen05.ld from TMEM, optional split-K reduction
// in the last-arriving CTA). For A_NF4_K the dequantized operand goes straight into
// tensor memory with tcgen05.st and the MMA reads A from there (likewise for
// A_CHANQ_K); the other sources stage A in shared memory. Every wait is bounded; on timeout the kernel records an
// error, stops, drains its own copies and MMAs, frees TMEM and returns.
#pragma once
#include "common.cuh"

namespace qnf4 {

enum : int { A_NF4_K = 0, A_NF4_MN = 1, A_DENSE_K = 2, A_DENSE_MN = 3, A_CHANQ_K = 4 };
enum : int { EPI_BF16 = 0, EPI_F32 = 1, EPI_UV = 2 };

constexpr int kRowsTile = 128;
constexpr int kStep = 64;
constexpr uint32_t kATile = 128u * 128u;  // 128 rows x 64 bf16 (or 2 x 64 x 64 MN-major)
constexpr uint32_t kPTile = 4096u;         // packed NF4 bytes of one step
constexpr int kMaxS1 = 16;
constexpr int kMaxS2 = 8;

__host__ __device__ constexpr bool src_deq(int a) {
  return a == A_NF4_K || a == A_NF4_MN || a == A_CHANQ_K;
}
__host__ __device__ constexpr bool src_mn(int a) { return a == A_NF4_MN || a == A_DENSE_MN; }
__host__ __device__ constexpr bool src_dense(int a) { return a == A_DENSE_K || a == A_DENSE_MN; }
__host__ __device__ constexpr bool src_packed_tma(int a) { return a == A_NF4_K || a == A_NF4_MN; }
// A operand staged in tensor memory (written by tcgen05.st) instead of shared memory
#ifndef QNF4_NF4K_TMEM_A
#define QNF4_NF4K_TMEM_A 1
#endif
__host__ __device__ constexpr bool src_tmem_a(int a) {
  return QNF4_NF4K_TMEM_A && (a == A_NF4_K || a == A_CHANQ_K);
}
__host__ __device__ constexpr int gemm_threads(int nset) { return 64 + 128 * nset; }

// TMEM columns: the fp32 accumulator (a power of two >= tn, at least 32), then
// (for A in tensor memory) s2 stages of 32 columns, one 128 x 64 bf16 A tile each.
__host__ __device__ inline uint32_t acc_cols(int tn) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(tn)) c <<= 1;
  return c;
}
__host__ __device__ inline uint32_t tmem_cols(int asrc, int tn, int s2) {
  uint32_t need = acc_cols(tn) + (src_tmem_a(asrc) ? 32u * static_cast<uint32_t>(s2) : 0u);
  uint32_t c = 32;
  while (c < need) c <<= 1;
  return c;
}

struct GemmArgs {
  int64_t rows, cols;     // extents of D
  int nsteps;             // contraction steps of 64 in total
  int steps_per_split;    // steps per blockIdx.z slice
  int splits;             // gridDim.z
  int tn;                 // N tile: multiple of 16, 16..256
  int s1, s2;             // depth of the load ring and of the dequantized-A ring
  int has_ext;            // add the adapter chunk (in split 0)
  int ext_k16;            // K=16 sub-steps of the adapter chunk (ceil(r/16))
  int ext_r;              // adapter rank r
  const uint16_t* ext_a;  // B [rows, r] (K-major chunk) or A [r, K] (MN-major chunk)
  int64_t ext_ld;         // row stride of ext_a in elements
  // two-level NF4 constants
  const uint8_t* code2;
  const float* scale2;
  const float* mean;
  int64_t nbk;            // 64-blocks per weight row (K / 64)
  int64_t wN;             // weight rows (output features)
  float levels[16];
  // per-channel quantizer
  const uint8_t* cq_packed;
  const int64_t* cq_row_off;
  const uint8_t* cq_bits;
  const float* cq_map;
  const int64_t* cq_map_off;
  const float* cq_absmax;
  // epilogue
  int epi;
  void* out;
  int64_t o_rs, o_cs;     // element strides of out for row / col
  int64_t out_cols;       // columns written (EPI_F32)
  void* out2;             // EPI_UV: transposed copy, [col][row] with stride o2_ld
  int64_t o2_ld;
  float scale;
  float* part;            // split-K partial tiles
  unsigned int* counters; // split-K arrival counters (zero on entry, left zero)
  unsigned long long wait_ns;
  int lazy_dep;           // programmatic dependent launch: 0 = every thread waits for the
                          // previous grid after the prologue; 1 = only the adapter chunk's
                          // copy waits (its operand is the one the previous grid writes)
};

struct SmemPlan {
  uint32_t off_a1, off_b1, off_p1, slot1, slot2, ring2, ext, cq, total;
};

__host__ __device__ inline SmemPlan smem_plan(int asrc, int tn, int s1, int s2, int has_ext) {
  SmemPlan p{};
  uint32_t o = 0;
  p.off_a1 = o;
  if (src_dense(asrc)) o += kATile;
  p.off_b1 = o;
  o += static_cast<uint32_t>(tn) * 128u;
  p.off_p1 = o;
  if (src_packed_tma(asrc)) o += kPTile;
  p.slot1 = (o + 1023u) & ~1023u;
  p.slot2 = (src_deq(asrc) && !src_tmem_a(asrc)) ? kATile : 0u;
  p.ring2 = static_cast<uint32_t>(s1) * p.slot1;
  p.ext = p.ring2 + static_cast<uint32_t>(s2) * p.slot2;
  p.cq = p.ext + (has_ext ? kATile : 0u);
  p.total = p.cq + (asrc == A_CHANQ_K ? 256u * 4u : 0u);
  return p;
}

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
#ifdef QNF4_WAIT_STATS
// Tracing build only: clock cycles spent blocked at each wait site (index = site,
// 0..63), summed over all threads that wait there. Read with qnf4_debug_wait_stats.
__device__ unsigned long long g_wait_cycles[64];
#endif

QNF4_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, unsigned long long wait_ns,
                            volatile int* abort_flag, unsigned int site) {
  if (mbar_try_wait(bar, parity)) return true;
#ifdef QNF4_WAIT_STATS
  const long long c0 = clock64();
  struct Acc {
    long long c0;
    unsigned int site;
    QNF4_DEV ~Acc() { atomicAdd(&g_wait_cycles[site & 63], static_cast<unsigned long long>(clock64() - c0)); }
  } acc{c0, site};
#endif
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > wait_ns) {
      set_err(site);
      *abort_flag = 1;
      return false;
    }
  }
}

QNF4_DEV void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Write one 128-byte row slot (64 bf16 given as 32 packed words) of a SW128 tile:
// 16-byte chunk c of row t lands at chunk position c ^ (t & 7).
QNF4_DEV void store_row_sw128(uint8_t* tile, int t, const uint32_t (&w)[32]) {
  uint8_t* row = tile + t * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 v = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    *reinterpret_cast<uint4*>(row + ((c ^ (t & 7)) << 4)) = v;
  }
}

// Register-resident NF4 lookup. For one block with constant c, the 16 possible
// dequantized values P[k] = bf16(fp32(levels[k] * c)) are computed once and split
// into byte planes: l[j] / h[j] hold the low / high bytes of P[4j .. 4j+3]. A
// byte-permute with a 3-bit selector then reads one plane entry per output byte,
// a second permute picks the 0-7 or 8-15 half by the code's top bit, and a third
// interleaves low and high bytes into bf16 pairs. The result equals rounding each
// fp32 product q[code] * c to bf16, the dequantization the QLoRA page describes.
struct Nf4Planes {
  uint32_t l[4], h[4];
};

QNF4_DEV void nf4_planes(const float (&lv)[16], float c, Nf4Planes& P) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = pack_bf16x2(lv[2 * i] * c, lv[2 * i + 1] * c);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    P.l[j] = __byte_perm(p[2 * j], p[2 * j + 1], 0x6420);
    P.h[j] = __byte_perm(p[2 * j], p[2 * j + 1], 0x7531);
  }
}

// 8 codes (one packed word: element 2j in the high nibble of byte j) -> 4 bf16 pairs
// (element 2j in the low half of o[j]).
QNF4_DEV void nf4_lookup8(uint32_t w, const Nf4Planes& P, uint32_t* o) {
  const uint32_t sa = w & 0x77777777u;
  const uint32_t sb = sa >> 16;
  const uint32_t ta = ((w >> 1) & 0x4444u) | 0x3210u;
  const uint32_t tb = ((w >> 17) & 0x4444u) | 0x3210u;
  const uint32_t la = __byte_perm(__byte_perm(P.l[0], P.l[1], sa), __byte_perm(P.l[2], P.l[3], sa), ta);
  const uint32_t ha = __byte_perm(__byte_perm(P.h[0], P.h[1], sa), __byte_perm(P.h[2], P.h[3], sa), ta);
  const uint32_t lb = __byte_perm(__byte_perm(P.l[0], P.l[1], sb), __byte_perm(P.l[2], P.l[3], sb), tb);
  const uint32_t hb = __byte_perm(__byte_perm(P.h[0], P.h[1], sb), __byte_perm(P.h[2], P.h[3], sb), tb);
  o[0] = __byte_perm(la, ha, 0x4051);
  o[1] = __byte_perm(la, ha, 0x6273);
  o[2] = __byte_perm(lb, hb, 0x4051);
  o[3] = __byte_perm(lb, hb, 0x6273);
}

// Dequantize one NF4 block: 32 packed bytes at src (shared memory) times constant c.
QNF4_DEV void nf4_block_to_bf16(const uint8_t* src, float c, const float (&lv)[16],
                                uint32_t (&o)[32]) {
  const uint4 a = *reinterpret_cast<const uint4*>(src);
  const uint4 b = *reinterpret_cast<const uint4*>(src + 16);
  Nf4Planes P;
  nf4_planes(lv, c, P);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) nf4_lookup8(w[i], P, &o[4 * i]);
}

QNF4_DEV void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

QNF4_DEV uint16_t f2bf(float f) {
  return static_cast<uint16_t>(pack_bf16x2(f, 0.f) & 0xFFFFu);
}

QNF4_DEV void epi_store(const GemmArgs& g, int64_t row, int64_t col0, const float* v, int n) {
  if (row >= g.rows) return;
  if (g.epi == EPI_BF16) {
    uint16_t* o = static_cast<uint16_t*>(g.out);
    for (int j = 0; j < n; ++j) {
      const int64_t col = col0 + j;
      if (col < g.cols) o[row * g.o_rs + col * g.o_cs] = f2bf(v[j]);
    }
  } else if (g.epi == EPI_F32) {
    float* o = static_cast<float*>(g.out);
    for (int j = 0; j < n; ++j) {
      const int64_t col = col0 + j;
      if (col < g.out_cols) o[row * g.o_rs + col * g.o_cs] = v[j] * g.scale;
    }
  } else {  // EPI_UV: rows are tokens, cols the adapter rank (padded)
    uint16_t* p = static_cast<uint16_t*>(g.out);
    uint16_t* pt = static_cast<uint16_t*>(g.out2);
    for (int j = 0; j < n; ++j) {
      const int64_t col = col0 + j;
      const uint16_t b = f2bf(v[j] * g.scale);
      if (p) p[row * 64 + col] = b;
      if (pt) pt[col * g.o2_ld + row] = b;
    }
  }
}

// Where a converter set's step i sits in the two rings, advanced without division
// (NSET < S2 <= S1, so an index wraps at most once per advance): s / ph = load-ring
// slot and phase of step i, s2 = its A stage, sj / phj = load-ring slot and phase of
// step i - S2, the last reader of that A stage (valid once i >= S2).
struct ConvCursor {
  int i, s, s2, sj;
  uint32_t ph, phj;
  QNF4_DEV explicit ConvCursor(int set) : i(set), s(set), s2(set), sj(0), ph(0), phj(0) {}
  QNF4_DEV void next(int nset, int S1, int S2) {
    i += nset;
    s += nset;
    if (s >= S1) {
      s -= S1;
      ph ^= 1u;
    }
    s2 += nset;
    if (s2 >= S2) s2 -= S2;
    const int j = i - S2;
    if (j >= 0) {
      if (j < nset) {  // first step with a predecessor: j < nset < S1
        sj = j;
        phj = 0;
      } else {
        sj += nset;
        if (sj >= S1) {
          sj -= S1;
          phj ^= 1u;
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int ASRC, int NSET, int MINB>
__global__ void __launch_bounds__(gemm_threads(NSET), MINB)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmBx, const GemmArgs g) {
  constexpr bool DEQ = src_deq(ASRC);
  constexpr bool MN = src_mn(ASRC);
  constexpr bool TMA_A = src_tmem_a(ASRC);
  constexpr int NCONV = 128 * NSET;  // converter / epilogue threads
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full1[kMaxS1], empty1[kMaxS1], full2[kMaxS2];
  __shared__ __align__(8) uint64_t acc_bar, ext_bar, fin_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_last;
  __shared__ float s_lv[16];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const SmemPlan sp = smem_plan(ASRC, g.tn, g.s1, g.s2, g.has_ext);
  const int S1 = g.s1, S2 = g.s2;
  const int z = blockIdx.z;
  const int step0 = z * g.steps_per_split;
  const int nst = max(0, min(g.nsteps - step0, g.steps_per_split));
  const bool ext = g.has_ext && z == 0;
  const int nload = nst + (ext ? 1 : 0);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kRowsTile;
  const int64_t col0 = static_cast<int64_t>(blockIdx.y) * g.tn;
  const uint32_t ncols = tmem_cols(ASRC, g.tn, S2);
#ifdef QNF4_WAIT_STATS
  const long long g_t_start = clock64();
#endif
  const uint32_t a_col = acc_cols(g.tn);  // first TMEM column of the A stages

  if (threadIdx.x == 0) {
    for (int i = 0; i < S1; ++i) {
      mbar_init(&full1[i], 1);
      mbar_init(&empty1[i], 1);
    }
    for (int i = 0; i < S2; ++i) mbar_init(&full2[i], 128);
    mbar_init(&acc_bar, 1);
    mbar_init(&ext_bar, 128);
    mbar_init(&fin_bar, 1);
    s_abort = 0;
    s_last = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) s_lv[threadIdx.x] = g.levels[threadIdx.x];
  if (warp == 1) {
    tmem_alloc(&s_tmem, ncols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    if (src_dense(ASRC) || src_packed_tma(ASRC)) tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (ext) tma_prefetch_desc(&tmBx);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // Programmatic dependent launch: the prologue above overlapped the previous grid.
  // Every kernel of the library waits for its predecessor before it lets its own
  // dependents start, so a dependent may read anything older than its predecessor.
  if (!g.lazy_dep) griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;
      int32_t kc = step0 * kStep;
      uint32_t bytes = static_cast<uint32_t>(g.tn) * 128u;
      if (src_dense(ASRC)) bytes += kATile;
      if (src_packed_tma(ASRC)) bytes += kPTile;
      for (int i = 0; i < nload; ++i) {
        if (!mbar_try_wait(&empty1[s], ph ^ 1) &&
            !wait_or_abort(&empty1[s], ph ^ 1, g.wait_ns, &s_abort, 11))
          break;
        uint8_t* slot = base + s * sp.slot1;
        uint64_t* fb = &full1[s];
        if (i < nst) {
          mbar_expect_tx(fb, bytes);
          if (ASRC == A_DENSE_K) tma_load_2d(slot + sp.off_a1, &tmA, fb, kc, (int32_t)row0);
          if (ASRC == A_DENSE_MN) {
            tma_load_2d(slot + sp.off_a1, &tmA, fb, (int32_t)row0, kc);
            tma_load_2d(slot + sp.off_a1 + 8192, &tmA, fb, (int32_t)row0 + 64, kc);
          }
          if (ASRC == A_NF4_K) tma_load_2d(slot + sp.off_p1, &tmA, fb, kc / 2, (int32_t)row0);
          if (ASRC == A_NF4_MN) tma_load_2d(slot + sp.off_p1, &tmA, fb, (int32_t)(row0 / 2), kc);
          tma_load_2d(slot + sp.off_b1, &tmB, fb, kc, (int32_t)col0);
        } else {
          if (g.lazy_dep) griddep_wait();
          mbar_expect_tx(fb, static_cast<uint32_t>(g.tn) * 128u);
          tma_load_2d(slot + sp.off_b1, &tmBx, fb, 0, (int32_t)col0);
        }
        issued = i + 1;
        kc += kStep;
        if (++s == S1) {
          s = 0;
          ph ^= 1;
        }
      }
      // Drain: the last copy issued into each slot must land before the CTA exits.
      // One deadline covers the whole drain.
      const int nslots = min(issued, S1);
      const uint64_t t0 = globaltimer();
      bool late = false;
      for (int s = 0; s < nslots && !late; ++s) {
        const int j = s + S1 * ((issued - 1 - s) / S1);
        while (!mbar_try_wait(&full1[s], (j / S1) & 1)) {
          if (globaltimer() - t0 > g.wait_ns) {
            set_err(12);
            late = true;
            break;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One thread keeps the tensor core fed: the descriptors are built once and only
    // offset per stage, stage indices and phases advance incrementally, and a step
    // costs one barrier test, four MMAs and one commit (the stage's release).
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, static_cast<uint32_t>(g.tn), MN ? 1u : 0u, 0u);
      const uint64_t bdesc0 = smem_desc(smem_u32(base + sp.off_b1), 16, 1024, kLayoutSW128);
      const uint32_t a_base = DEQ ? smem_u32(base + sp.ring2) : smem_u32(base + sp.off_a1);
      const uint64_t adesc0 = MN ? smem_desc(a_base, 8192, 1024, kLayoutSW128)
                                 : smem_desc(a_base, 16, 1024, kLayoutSW128);
      const uint32_t b_stride = sp.slot1 >> 4;                 // descriptor units per ring-1 slot
      const uint32_t a_stride = (DEQ ? sp.slot2 : sp.slot1) >> 4;
      constexpr uint32_t a_kstep = MN ? (2048u >> 4) : (32u >> 4);  // one K=16 sub-step
      const uint32_t tmem_a0 = tmem + a_col;
      bool ok = true;
      int s = 0, s2 = 0;
      uint32_t ph = 0, ph2 = 0;
      for (int i = 0; i < nst; ++i) {
        uint64_t* bar = DEQ ? &full2[s2] : &full1[s];
        const uint32_t pp = DEQ ? ph2 : ph;
        if (!mbar_try_wait(bar, pp) && !wait_or_abort(bar, pp, g.wait_ns, &s_abort, DEQ ? 22 : 21)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bd = bdesc0 + static_cast<uint64_t>(static_cast<uint32_t>(s) * b_stride);
        const uint64_t ad = adesc0 + static_cast<uint64_t>(static_cast<uint32_t>(DEQ ? s2 : s) * a_stride);
        const uint32_t ta = tmem_a0 + 32u * static_cast<uint32_t>(s2);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          if (TMA_A) mma_ts(tmem, ta + 8u * kk, bd + 2u * kk, idesc, acc);
          else mma_ss(tmem, ad + a_kstep * kk, bd + 2u * kk, idesc, acc);
        }
        mma_commit(&empty1[s]);  // frees ring-1 slot s and, S2 steps later, A stage s2
        if (++s == S1) {
          s = 0;
          ph ^= 1;
        }
        if (DEQ && ++s2 == S2) {
          s2 = 0;
          ph2 ^= 1;
        }
      }
      if (ok && ext) {
        const int i = nst;
        const int s = i % S1;
        if (wait_or_abort(&full1[s], (i / S1) & 1, g.wait_ns, &s_abort, 23) &&
            wait_or_abort(&ext_bar, 0, g.wait_ns, &s_abort, 24)) {
          tc_fence_after();
          const uint32_t aa = smem_u32(base + sp.ext);
          const uint32_t bb = smem_u32(base + s * sp.slot1 + sp.off_b1);
          for (int kk = 0; kk < g.ext_k16; ++kk) {
            const uint64_t ad = MN ? smem_desc(aa + kk * 2048, 8192, 1024, kLayoutSW128)
                                   : smem_desc(aa + kk * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd = smem_desc(bb + kk * 32, 16, 1024, kLayoutSW128);
            mma_ss(tmem, ad, bd, idesc, (nst > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty1[s]);
        }
      }
      mma_commit(&acc_bar);
      // Drain: every MMA of this CTA completes before TMEM and smem are released.
      mma_commit(&fin_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&fin_bar, 0)) {
        if (globaltimer() - t0 > g.wait_ns) {
          set_err(25);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - 64;  // 0 .. NCONV-1
    const int set = ct >> 7;          // converter set: steps i with i % NSET == set
    const int t = ct & 127;           // row slot 0..127
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    if (ext && set == 0) {
      uint32_t w[32];
      if (!MN) {
        // row slot t = D row (row0 + t): adapter B[row, 0..r), zero padded to 64
        const int64_t row = row0 + t;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int j0 = 2 * c;
          uint32_t lo = 0, hi = 0;
          if (row < g.rows) {
            if (j0 < g.ext_r) lo = g.ext_a[row * g.ext_ld + j0];
            if (j0 + 1 < g.ext_r) hi = g.ext_a[row * g.ext_ld + j0 + 1];
          }
          w[c] = lo | (hi << 16);
        }
      } else {
        // MN-major: row slot t = (atom kb, contraction j); A[j, row0 + 64 kb .. +64)
        const int kb = t >> 6, j = t & 63;
        const int64_t k0 = row0 + kb * 64;
        if (j < g.ext_r && k0 < g.rows) {
          const uint4* src = reinterpret_cast<const uint4*>(g.ext_a + j * g.ext_ld + k0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = src[c];
            w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) w[c] = 0u;
        }
      }
      store_row_sw128(base + sp.ext, t, w);
      fence_proxy_async();
      mbar_arrive(&ext_bar);
    }

    if constexpr (ASRC == A_NF4_K || ASRC == A_NF4_MN) {
      float lv[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) lv[k] = s_lv[k];
      const float mu = *g.mean;
      // In tensor memory the row slot must be the lane this warp may access.
      const int slot = TMA_A ? (q * 32 + lane) : t;
      ConvCursor cur(set);
      // block index of this slot at step i and its per-step increment
      int64_t bidx;
      int64_t bstep;
      bool rowok;
      if (ASRC == A_NF4_K) {
        const int64_t n = row0 + slot;
        rowok = n < g.wN;
        bidx = n * g.nbk + step0 + set;
        bstep = NSET;
      } else {
        const int kb = slot >> 6, nr = slot & 63;
        const int64_t kblk = row0 / 64 + kb;
        rowok = kblk < g.nbk;
        bidx = (static_cast<int64_t>(step0 + set) * kStep + nr) * g.nbk + kblk;
        bstep = static_cast<int64_t>(NSET) * kStep * g.nbk;
      }
      const int64_t nb1 = g.wN * g.nbk;
      // constants of this set's next step, fetched one of its steps ahead
      int64_t bnext = bidx;
      bool vnext = rowok && set < nst && bnext < nb1;
      uint32_t cnext = vnext ? g.code2[bnext] : 0u;
      float snext = vnext ? __ldg(g.scale2 + (bnext >> 8)) : 0.f;
      for (; cur.i < nst; cur.next(NSET, S1, S2)) {
        const int i = cur.i;
        const int s = cur.s, s2 = cur.s2;
        const bool valid = vnext;
        const float ch = valid ? fmaf(e4m3_to_f32(static_cast<uint8_t>(cnext)), snext, mu) : 0.f;
        bnext += bstep;
        vnext = rowok && (i + NSET) < nst && bnext < nb1;
        if (vnext) {
          cnext = g.code2[bnext];
          snext = __ldg(g.scale2 + (bnext >> 8));
        }
        if (!wait_or_abort(&full1[s], cur.ph, g.wait_ns, &s_abort, 31)) break;
        // A stage s2 was last read by step i - S2; its commit released load-ring slot
        // cur.sj in phase cur.phj. Waiting for that phase means the stage is free again.
        if (i >= S2 && !wait_or_abort(&empty1[cur.sj], cur.phj, g.wait_ns, &s_abort, 32)) break;
        const uint8_t* pk = base + s * sp.slot1 + sp.off_p1;
        const uint8_t* src =
            (ASRC == A_NF4_K) ? pk + slot * 32 : pk + (slot & 63) * 64 + (slot >> 6) * 32;
        uint32_t o[32];
        nf4_block_to_bf16(src, ch, lv, o);
        if (TMA_A) {
          tc_fence_after();
          tmem_st32(tmem + (static_cast<uint32_t>(q * 32) << 16) + a_col + 32u * s2, o);
          tmem_wait_st();
          tc_fence_before();
        } else {
          store_row_sw128(base + sp.ring2 + s2 * sp.slot2, slot, o);
          fence_proxy_async();
        }
        mbar_arrive(&full2[s2]);
      }
    } else if constexpr (ASRC == A_CHANQ_K) {
      // Row slot = the TMEM lane this warp may access; the row's 2^b mapping values
      // live in registers (unused entries 0), and each 64-element group's codes are
      // widened to the 4-bit layout of NF4 so the same register lookup applies.
      const int slot = q * 32 + lane;
      const int64_t n = row0 + slot;
      const bool valid = n < g.wN;
      uint32_t* s_t1 = reinterpret_cast<uint32_t*>(base + sp.cq);  // 1-bit byte -> nibble word
      if (set == 0) {
        for (int e = t; e < 256; e += 128) {
          uint32_t word = 0;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t hi = (static_cast<uint32_t>(e) >> (7 - 2 * m)) & 1u;
            const uint32_t lo = (static_cast<uint32_t>(e) >> (6 - 2 * m)) & 1u;
            word |= ((hi << 4) | lo) << (8 * m);
          }
          s_t1[e] = word;
        }
      }
      named_sync(2, NCONV);  // the table is read by every converter set
      int bits = 1;
      const uint8_t* prow = nullptr;
      float mp[16];
      {
        int64_t mo = 0;
        if (valid) {
          bits = g.cq_bits[n];
          prow = g.cq_packed + g.cq_row_off[n];
          mo = g.cq_map_off[n];
        }
        const int nmap = valid ? (1 << bits) : 0;
#pragma unroll
        for (int c = 0; c < 16; ++c) mp[c] = c < nmap ? g.cq_map[mo + c] : 0.f;
      }
      for (ConvCursor cur(set); cur.i < nst; cur.next(NSET, S1, S2)) {
        const int i = cur.i;
        const int s2 = cur.s2;
        const int gi = step0 + i;
        // the group's codes and scale (issued before the waits)
        uint32_t cw[8];
        float gm = 0.f;
        if (valid) {
          gm = __ldg(g.cq_absmax + n * g.nbk + gi);
          // A row holds K b / 8 bytes (a multiple of 8, not of 16, e.g. K = 448) and a
          // group 8 b bytes, so only 8-byte loads are aligned for every shape.
          const uint2* src = reinterpret_cast<const uint2*>(prow + static_cast<int64_t>(gi) * 8 * bits);
          if (bits == 4) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint2 a = __ldg(src + k);
              cw[2 * k] = a.x;
              cw[2 * k + 1] = a.y;
            }
          } else if (bits == 2) {
            const uint2 a0 = __ldg(src), a1 = __ldg(src + 1);
            const uint32_t in[4] = {a0.x, a0.y, a1.x, a1.y};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // byte x = c0 c1 c2 c3 (2 bits each, first at the top) -> (c0 c1), (c2 c3)
              const uint32_t w = in[k];
              const uint32_t hi = ((w >> 2) & 0x30303030u) | ((w >> 4) & 0x03030303u);
              const uint32_t lo = ((w << 2) & 0x30303030u) | (w & 0x03030303u);
              cw[2 * k] = __byte_perm(hi, lo, 0x5140);
              cw[2 * k + 1] = __byte_perm(hi, lo, 0x7362);
            }
          } else {
            const uint2 a = __ldg(src);
#pragma unroll
            for (int k = 0; k < 8; ++k) cw[k] = s_t1[((k < 4 ? a.x : a.y) >> (8 * (k & 3))) & 0xFFu];
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) cw[k] = 0u;
        }
        if (!wait_or_abort(&full1[cur.s], cur.ph, g.wait_ns, &s_abort, 33)) break;
        if (i >= S2 && !wait_or_abort(&empty1[cur.sj], cur.phj, g.wait_ns, &s_abort, 34)) break;
        uint32_t o[32];
        Nf4Planes P;
        nf4_planes(mp, gm, P);
#pragma unroll
        for (int k = 0; k < 8; ++k) nf4_lookup8(cw[k], P, &o[4 * k]);
        if (TMA_A) {
          tc_fence_after();
          tmem_st32(tmem + (static_cast<uint32_t>(q * 32) << 16) + a_col + 32u * s2, o);
          tmem_wait_st();
          tc_fence_before();
        } else {
          store_row_sw128(base + sp.ring2 + s2 * sp.slot2, slot, o);
          fence_proxy_async();
        }
        mbar_arrive(&full2[s2]);
      }
    }

    // ------------------------------------------------------------ epilogue
    // The decision to write is taken once, so all converter threads take the same
    // path through the named barriers below.
    wait_or_abort(&acc_bar, 0, g.wait_ns, &s_abort, 41);
    named_sync(1, NCONV);
    if (ct == 0) s_last = s_abort ? 0 : 2;
    named_sync(1, NCONV);
    const bool have = s_last == 2;
    named_sync(1, NCONV);
    tc_fence_after();
    const int rl = q * 32 + lane;
    const int64_t row = row0 + rl;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    // the sets split the tile's columns in 16-column chunks
    const int nchunk = g.tn / 16;
    if (have) {
      if (g.splits == 1) {
        for (int ck = set; ck < nchunk; ck += NSET) {
          const int c0 = ck * 16;
          uint32_t r[16];
          tmem_ld16(taddr + c0, r);
          tmem_wait_ld();
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
          epi_store(g, row, col0 + c0, v, 16);
        }
      } else {
        const int64_t tile = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
        const int64_t tsz = static_cast<int64_t>(g.tn) * 128;
        float* mine = g.part + (tile * g.splits + z) * tsz;
        for (int ck = set; ck < nchunk; ck += NSET) {
          const int c0 = ck * 16;
          uint32_t r[16];
          tmem_ld16(taddr + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) __stcg(mine + (c0 + j) * 128 + rl, __uint_as_float(r[j]));
        }
        __threadfence();
        named_sync(1, NCONV);
        if (ct == 0) {
          const unsigned int old = atomicAdd(g.counters + tile, 1u);
          s_last = (old == static_cast<unsigned int>(g.splits - 1)) ? 1 : 0;
        }
        named_sync(1, NCONV);
        if (s_last) {
          __threadfence();
          const float* all = g.part + tile * g.splits * tsz;
          for (int ck = set; ck < nchunk; ck += NSET) {
            const int c0 = ck * 16;
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
            // Partials in split order (deterministic), four splits' loads in flight at
            // a time so the reduction costs one L2 round trip per four splits.
            for (int zz = 0; zz < g.splits; zz += 4) {
              float t[4][16];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const bool in = zz + u < g.splits;
                const float* src = all + (zz + u) * tsz + c0 * 128 + rl;
#pragma unroll
                for (int j = 0; j < 16; ++j) t[u][j] = in ? __ldcg(src + j * 128) : 0.f;
              }
#pragma unroll
              for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] += t[u][j];
              }
            }
            epi_store(g, row, col0 + c0, v, 16);
          }
          if (ct == 0) g.counters[tile] = 0u;
        }
      }
    }
    tc_fence_before();
  }

#ifdef QNF4_WAIT_STATS
  if (lane == 0) {
    // per-warp active time: 60 = producer, 61 = MMA, 62 = converters (sum of warps)
    const unsigned int slot = warp == 0 ? 60 : (warp == 1 ? 61 : 62);
    atomicAdd(&g_wait_cycles[slot], static_cast<unsigned long long>(clock64() - g_t_start));
  }
#endif
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// Transpose the adapter B [N, r] (bf16) into BT [r, ldn] so it can serve as a
// K-major TMA operand of v = dY B.
__global__ void __launch_bounds__(256) k_transpose_b(const uint16_t* __restrict__ B, int64_t N,
                                                     int r, uint16_t* __restrict__ BT,
                                                     int64_t ldn) {
  const int64_t total = N * r;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = i / N, n = i - j * N;
    BT[j * ldn + n] = B[n * r + j];
  }
}

}  // namespace qnf4
