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
//   A_CHANQ_MN the same weight read transposed (backward dX), from codes widened to
//              the NF4 nibble layout beforehand: TMA brings each step's code tile and
//              its 64 rows' 16-entry tables; the converters look up like A_NF4_MN.
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

enum : int { A_NF4_K = 0, A_NF4_MN = 1, A_DENSE_K = 2, A_DENSE_MN = 3, A_CHANQ_K = 4, A_CHANQ_MN = 5 };
enum : int { EPI_BF16 = 0, EPI_F32 = 1, EPI_UV = 2 };

constexpr int kRowsTile = 128;
constexpr int kStep = 64;
constexpr uint32_t kATile = 128u * 128u;  // 128 rows x 64 bf16 (or 2 x 64 x 64 MN-major)
constexpr uint32_t kPTile = 4096u;         // packed NF4 bytes of one step
constexpr int kMaxS1 = 16;
constexpr int kMaxS2 = 8;

__host__ __device__ constexpr bool src_deq(int a) {
  return a == A_NF4_K || a == A_NF4_MN || a == A_CHANQ_K || a == A_CHANQ_MN;
}
__host__ __device__ constexpr bool src_mn(int a) {
  return a == A_NF4_MN || a == A_DENSE_MN || a == A_CHANQ_MN;
}
__host__ __device__ constexpr bool src_dense(int a) { return a == A_DENSE_K || a == A_DENSE_MN; }
__host__ __device__ constexpr bool src_packed_tma(int a) {
  return a == A_NF4_K || a == A_NF4_MN || a == A_CHANQ_MN;
}
// a per-step tile of 64 rows' 16-entry fp32 mapping tables (4 KB) rides in the load ring
__host__ __device__ constexpr bool src_table_tma(int a) { return a == A_CHANQ_MN; }
constexpr uint32_t kTTile = 64u * 16u * 4u;
// A operand staged in tensor memory (written by tcgen05.st) instead of shared memory
__host__ __device__ constexpr bool src_tmem_a(int a) { return a == A_NF4_K || a == A_CHANQ_K; }
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
  // Work units, taken by CTA b in the order b, b + gridDim.x, ...: units
  // 0 .. full_tiles-1 are whole tiles (tile t = unit), the following
  // tail_tiles * tail_splits units are contraction slices of the remaining tiles
  // (tile full_tiles + v % tail_tiles, slice v / tail_tiles, tail_sps steps each),
  // reduced by the last slice to finish. Tile t covers row tile t % row_tiles and
  // column tile t / row_tiles.
  int row_tiles;
  int full_tiles;
  int tail_tiles, tail_splits, tail_sps;
  int nunits;
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
  int stage;              // EPI_BF16 whole tiles leave through shared memory and the tmO
                          // tensor map (out rows contiguous, 16-byte row stride, has_ext)
  float* part;            // partial tiles of the tail slices [tail_tiles][tail_splits][tn][128]
  unsigned int* counters; // arrival counters per tail tile (zero on entry, left zero)
  unsigned long long wait_ns;
  // extents the checked build tests indices against (elements): out, out2, the partial
  // tiles, the arrival counters and the block constants (code2 or per-channel absmax)
  int64_t out_elems, out2_elems, part_elems, cnt_elems, cst_elems;
  const uint8_t* packed;  // A_NF4_K: the packed codes [wN, nbk * 32] (for the L2 prefetch)
  int lut;                // NF4 sources: copies of the shared-memory pair table (16 or 32;
                          // nf4_block_lut), 0 = the register byte planes
  int lazy_dep;           // programmatic dependent launch: 0 = every thread waits for the
                          // previous grid after the prologue; 1 = only the adapter chunk's
                          // copy waits (its operand is the one the previous grid writes)
};

struct SmemPlan {
  uint32_t off_a1, off_b1, off_p1, off_t1, slot1, slot2, ring2, ext, cq, lut, total;
};

// Shared-memory NF4 lookup table: one entry per packed byte value (the two bf16 levels
// the byte's nibbles select), replicated `copies` times (16 or 32) with lane l reading
// copy l mod copies: 32 copies never share a bank within a warp, 16 copies at most two
// lanes per bank (8 or 16 KB less shared memory).
__host__ __device__ constexpr uint32_t lut_bytes(int copies) { return 256u * static_cast<uint32_t>(copies) * 4u; }

__host__ __device__ inline SmemPlan smem_plan(int asrc, int tn, int s1, int s2, int has_ext,
                                              int lut = 0) {
  SmemPlan p{};
  uint32_t o = 0;
  p.off_a1 = o;
  if (src_dense(asrc)) o += kATile;
  p.off_b1 = o;
  o += static_cast<uint32_t>(tn) * 128u;
  p.off_p1 = o;
  if (src_packed_tma(asrc)) o += kPTile;
  p.off_t1 = o;
  if (src_table_tma(asrc)) o += kTTile;
  p.slot1 = (o + 1023u) & ~1023u;
  p.slot2 = (src_deq(asrc) && !src_tmem_a(asrc)) ? kATile : 0u;
  p.ring2 = static_cast<uint32_t>(s1) * p.slot1;
  p.ext = p.ring2 + static_cast<uint32_t>(s2) * p.slot2;
  p.cq = p.ext + (has_ext ? kATile : 0u);
  p.lut = p.cq + (asrc == A_CHANQ_K ? 256u * 4u : 0u);
  p.total = p.lut + ((lut && (asrc == A_NF4_K || asrc == A_NF4_MN)) ? lut_bytes(lut) : 0u);
  return p;
}

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
// Bounded wait; `lng` marks a long wait (producer slots, whole-tile MMAs), which lets
// the hardware suspend the thread between polls.
QNF4_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, unsigned long long wait_ns,
                            volatile int* abort_flag, unsigned int site, bool lng = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = wait_clock();
  while (true) {
    if (lng ? mbar_try_wait_long(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (wait_clock() - t0 > ns_cycles(wait_ns)) {
      set_err(site);
      *abort_flag = 1;
      return false;
    }
  }
}

QNF4_DEV void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Barrier of one converter set's 128 threads (ids 3 .. 3 + NSET - 1, immediates so the
// kernel reserves only the barriers it uses).
template <int NSET>
QNF4_DEV void set_sync(int set) {
  if (NSET == 1 || set == 0) asm volatile("bar.sync 3, 128;" ::: "memory");
  else if (NSET == 2 || set == 1) asm volatile("bar.sync 4, 128;" ::: "memory");
  else asm volatile("bar.sync 5, 128;" ::: "memory");
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

// Dequantize one NF4 block through the shared-memory pair table: each packed byte
// (element 2j in the high nibble) indexes the table entry holding bf16(q[hi]) and
// bf16(q[lo]); one packed bf16 multiply by the block constant c2 = (bf16(c), bf16(c))
// then gives bf16(bf16(q) bf16(c)) for both elements. The lane's table copy starts at
// shared address tb. Per two codes: one byte extract, one shared load, one multiply
// (the register byte-plane lookup spends about five integer operations there).
QNF4_DEV uint32_t lds_u32(uint32_t addr) {  // read-only table: not volatile
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
QNF4_DEV uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
QNF4_DEV void nf4_block_lut(const uint8_t* src, uint32_t c2, uint32_t tb, uint32_t sh,
                            uint32_t (&o)[32]) {
  const uint4 a = *reinterpret_cast<const uint4*>(src);
  const uint4 b = *reinterpret_cast<const uint4*>(src + 16);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t beta = __byte_perm(w[i], 0u, 0x4440u | static_cast<uint32_t>(j));
      o[4 * i + j] = hmul2_bf16(lds_u32(tb + (beta << sh)), c2);
    }
  }
}
// Fill the table (every thread of the CTA takes part; a CTA barrier must follow).
QNF4_DEV void lut_fill(uint32_t* tab, const float* s_lv, int copies, int tid, int nthreads) {
  for (int i = tid; i < 256 * copies; i += nthreads) {
    const int beta = i / copies;
    tab[i] = pack_bf16x2(s_lv[beta >> 4], s_lv[beta & 15]);
  }
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
      const int64_t at = row * g.o_rs + col * g.o_cs;
      if (col < g.cols && in_bounds(at < g.out_elems, 21)) o[at] = f2bf(v[j]);
    }
  } else if (g.epi == EPI_F32) {
    float* o = static_cast<float*>(g.out);
    for (int j = 0; j < n; ++j) {
      const int64_t col = col0 + j;
      const int64_t at = row * g.o_rs + col * g.o_cs;
      if (col < g.out_cols && in_bounds(at < g.out_elems, 21)) o[at] = v[j] * g.scale;
    }
  } else {  // EPI_UV: rows are tokens, cols the adapter rank (padded)
    uint16_t* p = static_cast<uint16_t*>(g.out);
    uint16_t* pt = static_cast<uint16_t*>(g.out2);
    for (int j = 0; j < n; ++j) {
      const int64_t col = col0 + j;
      const uint16_t b = f2bf(v[j] * g.scale);
      if (p && in_bounds(row * 64 + col < g.out_elems, 22)) p[row * 64 + col] = b;
      if (pt && in_bounds(col * g.o2_ld + row < g.out2_elems, 23)) pt[col * g.o2_ld + row] = b;
    }
  }
}

// One work unit: a tile of D and the contraction steps it covers.
struct Unit {
  int64_t row0, col0;  // first row / column of the tile
  int step0, nst;      // first contraction step and number of steps
  int z, splits;       // slice index and slices of this tile (1: a whole tile)
  int pt;              // tail tile index (partials and counter), when splits > 1
  bool ext;            // the adapter chunk is added here (slice 0)
};

QNF4_DEV Unit unit_of(const GemmArgs& g, int u) {
  Unit w;
  int t;
  int sps;
  if (u < g.full_tiles) {
    t = u;
    w.z = 0;
    w.splits = 1;
    w.pt = 0;
    sps = g.nsteps;
  } else {
    const int v = u - g.full_tiles;
    w.pt = v % g.tail_tiles;
    w.z = v / g.tail_tiles;
    t = g.full_tiles + w.pt;
    w.splits = g.tail_splits;
    sps = g.tail_sps;
  }
  const int rt = t % g.row_tiles;
  w.row0 = static_cast<int64_t>(rt) * kRowsTile;
  w.col0 = static_cast<int64_t>(t / g.row_tiles) * g.tn;
  w.step0 = w.z * sps;
  w.nst = max(0, min(g.nsteps - w.step0, sps));
  w.ext = g.has_ext && w.z == 0;
  return w;
}

// Where a converter set's step sits in the two rings, advanced without division
// (NSET <= S2 <= S1, so an index wraps at most once per advance). Both rings advance
// once per position, over all units of the CTA: a unit's contraction steps, then its
// adapter chunk. i = position in the unit, r = ring position, s / ph = load-ring slot
// and phase, s2 = A stage; sj / phj = load-ring slot and phase of position r - S2,
// the last user of that A stage (valid once r >= S2): the MMA's release of that slot
// also releases the stage.
struct ConvCursor {
  int i, r, s, s2, sj;
  uint32_t ph, phj;
  QNF4_DEV ConvCursor(int set, int rbase, int S1, int S2) {
    i = set;
    r = rbase + set;
    s = r % S1;
    ph = static_cast<uint32_t>(r / S1) & 1u;
    s2 = r % S2;
    const int j = r - S2;
    sj = j >= 0 ? j % S1 : 0;
    phj = j >= 0 ? (static_cast<uint32_t>(j / S1) & 1u) : 0u;
  }
  QNF4_DEV void next(int nset, int S1, int S2) {
    i += nset;
    r += nset;
    s += nset;
    if (s >= S1) {
      s -= S1;
      ph ^= 1u;
    }
    s2 += nset;
    if (s2 >= S2) s2 -= S2;
    const int j = r - S2;
    if (j >= 0) {
      if (j < nset) {  // first position with a predecessor: j < nset <= S1
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
// Persistent: CTA b runs units b, b + gridDim.x, ... The load and A rings and their
// phases continue from unit to unit; the accumulator is handed back and forth
// through acc_bar (MMAs of a unit done) and acc_empty (its epilogue has read TMEM).
template <int ASRC, int NSET, int MINB>
__global__ void __launch_bounds__(gemm_threads(NSET), MINB)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmO,
           const __grid_constant__ CUtensorMap tmT,
           const GemmArgs g) {
  constexpr bool DEQ = src_deq(ASRC);
  constexpr bool MN = src_mn(ASRC);
  constexpr bool TMA_A = src_tmem_a(ASRC);
  constexpr int NCONV = 128 * NSET;  // converter / epilogue threads
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full1[kMaxS1], empty1[kMaxS1], full2[kMaxS2];
  __shared__ __align__(8) uint64_t acc_bar, acc_empty, ext_bar, fin_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_last;
  __shared__ float s_lv[16];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const SmemPlan sp = smem_plan(ASRC, g.tn, g.s1, g.s2, g.has_ext, g.lut);
  const int S1 = g.s1, S2 = g.s2;
  const int u0 = blockIdx.x;
  const int ustep = gridDim.x;
  const uint32_t ncols = tmem_cols(ASRC, g.tn, S2);
  const uint32_t a_col = acc_cols(g.tn);  // first TMEM column of the A stages

  if (threadIdx.x == 0) {
    for (int i = 0; i < S1; ++i) {
      mbar_init(&full1[i], 1);
      mbar_init(&empty1[i], 1);
    }
    for (int i = 0; i < S2; ++i) mbar_init(&full2[i], 128);
    mbar_init(&acc_bar, 1);
    mbar_init(&acc_empty, NCONV);
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
    if (g.has_ext) tma_prefetch_desc(&tmBx);
    if (g.stage) tma_prefetch_desc(&tmO);
    if (src_table_tma(ASRC)) tma_prefetch_desc(&tmT);
  }
  if ((ASRC == A_NF4_K || ASRC == A_NF4_MN) && g.lut)
    lut_fill(reinterpret_cast<uint32_t*>(base + sp.lut), g.levels, g.lut, threadIdx.x, blockDim.x);
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
    // Decode tiles read 32 bytes of each of 128 rows per step, rows K/2 bytes apart:
    // first the whole warp asks L2 for every unit's row slices of this CTA (contiguous
    // per row), so DRAM streams whole row ranges instead of scattered 32-byte pieces.
    if (ASRC == A_NF4_K && g.tn <= 32 && g.packed) {
      for (int u = u0; u < g.nunits; u += ustep) {
        const Unit w = unit_of(g, u);
        if (w.nst <= 0) continue;
        for (int r = lane; r < kRowsTile; r += 32) {
          const int64_t row = w.row0 + r;
          if (row < g.wN)
            prefetch_l2(g.packed + row * g.nbk * 32 + static_cast<int64_t>(w.step0) * 32,
                        static_cast<uint32_t>(w.nst) * 32u);
        }
      }
      __syncwarp();
    }
    if (lane == 0) {
      int issued = 0;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true, dep = false;
      uint32_t bytes = static_cast<uint32_t>(g.tn) * 128u;
      if (src_dense(ASRC)) bytes += kATile;
      if (src_packed_tma(ASRC)) bytes += kPTile;
      if (src_table_tma(ASRC)) bytes += kTTile;
      for (int u = u0; u < g.nunits && ok; u += ustep) {
        const Unit w = unit_of(g, u);
        const int nload = w.nst + (w.ext ? 1 : 0);
        int32_t kc = w.step0 * kStep;
        for (int i = 0; i < nload; ++i) {
          if (!mbar_try_wait(&empty1[s], ph ^ 1) &&
              !wait_or_abort(&empty1[s], ph ^ 1, g.wait_ns, &s_abort, 11, true)) {
            ok = false;
            break;
          }
          uint8_t* slot = base + s * sp.slot1;
          uint64_t* fb = &full1[s];
          if (i < w.nst) {
            mbar_expect_tx(fb, bytes);
            if (ASRC == A_DENSE_K) tma_load_2d(slot + sp.off_a1, &tmA, fb, kc, (int32_t)w.row0);
            if (ASRC == A_DENSE_MN) {
              tma_load_2d(slot + sp.off_a1, &tmA, fb, (int32_t)w.row0, kc);
              tma_load_2d(slot + sp.off_a1 + 8192, &tmA, fb, (int32_t)w.row0 + 64, kc);
            }
            if (ASRC == A_NF4_K) tma_load_2d(slot + sp.off_p1, &tmA, fb, kc / 2, (int32_t)w.row0);
            if (ASRC == A_NF4_MN || ASRC == A_CHANQ_MN)
              tma_load_2d(slot + sp.off_p1, &tmA, fb, (int32_t)(w.row0 / 2), kc);
            // the tables of this step's 64 contraction rows
            if (ASRC == A_CHANQ_MN) tma_load_2d(slot + sp.off_t1, &tmT, fb, 0, kc);
            tma_load_2d(slot + sp.off_b1, &tmB, fb, kc, (int32_t)w.col0);
          } else {
            if (g.lazy_dep && !dep) {
              griddep_wait();
              dep = true;
            }
            mbar_expect_tx(fb, static_cast<uint32_t>(g.tn) * 128u);
            tma_load_2d(slot + sp.off_b1, &tmBx, fb, 0, (int32_t)w.col0);
          }
          ++issued;
          kc += kStep;
          if (++s == S1) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // Drain: the last copy issued into each slot must land before the CTA exits.
      // One deadline covers the whole drain.
      const int nslots = min(issued, S1);
      const long long t0 = wait_clock();
      bool late = false;
      for (int s = 0; s < nslots && !late; ++s) {
        const int j = s + S1 * ((issued - 1 - s) / S1);
        while (!mbar_try_wait_long(&full1[s], (j / S1) & 1)) {
          if (wait_clock() - t0 > ns_cycles(drain_ns(g.wait_ns))) {
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
    // costs one barrier test, four MMAs and the stage releases.
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
      int k = 0, kx = 0;  // units done, adapter chunks done
      for (int u = u0; u < g.nunits; u += ustep, ++k) {
        const Unit w = unit_of(g, u);
        // the previous unit's epilogue must have read the accumulator
        if (k > 0) {
          if (!wait_or_abort(&acc_empty, (k - 1) & 1, g.wait_ns, &s_abort, 26, true)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        for (int i = 0; i < w.nst; ++i) {
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
          // frees load-ring slot s and, for a dequantized A, A stage s2
          mma_commit(&empty1[s]);
          if (++s == S1) {
            s = 0;
            ph ^= 1;
          }
          if (DEQ && ++s2 == S2) {
            s2 = 0;
            ph2 ^= 1;
          }
        }
        if (!ok) break;
        if (w.ext) {
          // The adapter chunk: one more position of both rings. Its full2 arrival is
          // bookkeeping only; its B tile and A tile are waited for here.
          if ((DEQ && !wait_or_abort(&full2[s2], ph2, g.wait_ns, &s_abort, 22)) ||
              !wait_or_abort(&full1[s], ph, g.wait_ns, &s_abort, 23) ||
              !wait_or_abort(&ext_bar, kx & 1, g.wait_ns, &s_abort, 24)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bd = bdesc0 + static_cast<uint64_t>(static_cast<uint32_t>(s) * b_stride);
          const uint32_t aa = smem_u32(base + sp.ext);
          for (int kk = 0; kk < g.ext_k16; ++kk) {
            const uint64_t ad = MN ? smem_desc(aa + kk * 2048, 8192, 1024, kLayoutSW128)
                                   : smem_desc(aa + kk * 32, 16, 1024, kLayoutSW128);
            mma_ss(tmem, ad, bd + 2u * kk, idesc, (w.nst > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty1[s]);
          if (++s == S1) {
            s = 0;
            ph ^= 1;
          }
          if (DEQ && ++s2 == S2) {
            s2 = 0;
            ph2 ^= 1;
          }
          ++kx;
        }
        mma_commit(&acc_bar);
      }
      // Drain: every MMA of this CTA completes before TMEM and smem are released.
      mma_commit(&fin_bar);
      const long long t0 = wait_clock();
      while (!mbar_try_wait_long(&fin_bar, 0)) {
        if (wait_clock() - t0 > ns_cycles(drain_ns(g.wait_ns))) {
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
    const int lrow = q * 32 + lane;   // the accumulator row (TMEM lane) of this thread
    bool dead = false;                // a wait of this thread gave up

    // The adapter operand of unit w into the ext tile (converter set 0 only).
    auto write_ext = [&](const Unit& w) {
      uint32_t v[32];
      if (!MN) {
        // row slot t = D row (row0 + t): adapter B[row, 0..r), zero padded to 64
        const int64_t row = w.row0 + t;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int j0 = 2 * c;
          uint32_t lo = 0, hi = 0;
          if (row < g.rows) {
            if (j0 < g.ext_r) lo = g.ext_a[row * g.ext_ld + j0];
            if (j0 + 1 < g.ext_r) hi = g.ext_a[row * g.ext_ld + j0 + 1];
          }
          v[c] = lo | (hi << 16);
        }
      } else {
        // MN-major: row slot t = (atom kb, contraction j); A[j, row0 + 64 kb .. +64)
        const int kb = t >> 6, j = t & 63;
        const int64_t k0 = w.row0 + kb * 64;
        if (j < g.ext_r && k0 < g.rows) {
          const uint4* src = reinterpret_cast<const uint4*>(g.ext_a + j * g.ext_ld + k0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 x = src[c];
            v[4 * c] = x.x; v[4 * c + 1] = x.y; v[4 * c + 2] = x.z; v[4 * c + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = 0u;
        }
      }
      store_row_sw128(base + sp.ext, t, v);
      fence_proxy_async();
      mbar_arrive(&ext_bar);
    };

    // Epilogue of the k-th unit of this CTA. Every converter thread calls it for the
    // same units in the same order; it returns false for all of them alike once the
    // CTA has aborted, so all take the same path through the named barriers.
    auto epilogue = [&](int u, int k) -> bool {
      wait_or_abort(&acc_bar, k & 1, g.wait_ns, &s_abort, 41, true);
      named_sync(1, NCONV);
      if (ct == 0) s_last = s_abort ? 0 : 2;
      named_sync(1, NCONV);
      const bool have = s_last == 2;
      named_sync(1, NCONV);
      if (!have) return false;
      tc_fence_after();
      const Unit w = unit_of(g, u);
      const int64_t row = w.row0 + lrow;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      // the sets split the tile's columns in 16-column chunks
      const int nchunk = g.tn / 16;
      if (w.splits == 1 && g.stage) {
        // 8-column pieces (bf16, [8 columns][128 rows]) through two 2 KB buffers per
        // set in the adapter tile, which is idle from the unit's last MMA to the next
        // unit's adapter write; one thread of the set stores each piece by TMA.
        uint8_t* stg = base + sp.ext + set * 4096;
        const int npiece = g.tn / 8;
        int p = set;
        uint32_t r[8];
        if (p < npiece) tmem_ld8(taddr + p * 8, r);
        for (int b = 0; p < npiece; p += NSET, b ^= 1) {
          tmem_wait_ld();
          uint32_t v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = r[j];
          if (p + NSET < npiece) tmem_ld8(taddr + (p + NSET) * 8, r);  // next piece in flight
          uint16_t* dst = reinterpret_cast<uint16_t*>(stg + b * 2048) + lrow;
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j * 128] = f2bf(__uint_as_float(v[j]));
          fence_proxy_async();
          if (t == 0) bulk_wait_read0();  // the set's previous piece has left buffer b ^ 1
          set_sync<NSET>(set);
          if (t == 0) {
            tma_store_2d(&tmO, stg + b * 2048, static_cast<int32_t>(w.row0),
                         static_cast<int32_t>(w.col0 + p * 8));
            bulk_commit();
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty);
        // the adapter tile is free for its next write once every piece has left it
        if (t == 0) bulk_wait_read0();
        named_sync(1, NCONV);
      } else if (w.splits == 1) {
        for (int ck = set; ck < nchunk; ck += NSET) {
          const int c0 = ck * 16;
          uint32_t r[16];
          tmem_ld16(taddr + c0, r);
          tmem_wait_ld();
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
          epi_store(g, row, w.col0 + c0, v, 16);
        }
        tc_fence_before();
        mbar_arrive(&acc_empty);
      } else {
        const int64_t tsz = static_cast<int64_t>(g.tn) * 128;
        const int64_t mine_at = (static_cast<int64_t>(w.pt) * w.splits + w.z) * tsz;
        float* mine = g.part + mine_at;
        const bool part_ok = in_bounds(mine_at + tsz <= g.part_elems, 24);
        for (int ck = set; ck < nchunk; ck += NSET) {
          const int c0 = ck * 16;
          uint32_t r[16];
          tmem_ld16(taddr + c0, r);
          tmem_wait_ld();
          if (part_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) __stcg(mine + (c0 + j) * 128 + lrow, __uint_as_float(r[j]));
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty);
        __threadfence();
        named_sync(1, NCONV);
        if (ct == 0) {
          s_last = 0;
          if (in_bounds(w.pt < g.cnt_elems, 25)) {
            const unsigned int old = atomicAdd(g.counters + w.pt, 1u);
            s_last = (old == static_cast<unsigned int>(w.splits - 1)) ? 1 : 0;
          }
        }
        named_sync(1, NCONV);
        if (s_last) {
          __threadfence();
          const float* all = g.part + static_cast<int64_t>(w.pt) * w.splits * tsz;
          in_bounds((static_cast<int64_t>(w.pt) + 1) * w.splits * tsz <= g.part_elems, 26);
          // Pieces of RW columns: in the wide dequantizing kernels the next unit's
          // conversion state stays live across the epilogue within a tight register
          // budget, so their reduction takes 8 columns; the others take 16 (half the
          // L2 round trips of the last slice).
          constexpr int RW = (DEQ && NSET > 1) ? 8 : 16;
          for (int ck = set; ck < nchunk * (16 / RW); ck += NSET) {
            const int c0 = ck * RW;
            float v[RW];
#pragma unroll
            for (int j = 0; j < RW; ++j) v[j] = 0.f;
            // Partials in slice order (deterministic), four slices' loads in flight
            // at a time so the reduction costs one L2 round trip per four slices.
            for (int zz = 0; zz < w.splits; zz += 4) {
              float tt[4][RW];
#pragma unroll
              for (int uu = 0; uu < 4; ++uu) {
                const bool in = zz + uu < w.splits;
                const float* src = all + (zz + uu) * tsz + c0 * 128 + lrow;
#pragma unroll
                for (int j = 0; j < RW; ++j) tt[uu][j] = in ? __ldcg(src + j * 128) : 0.f;
              }
#pragma unroll
              for (int uu = 0; uu < 4; ++uu) {
#pragma unroll
                for (int j = 0; j < RW; ++j) v[j] += tt[uu][j];
              }
            }
            epi_store(g, row, w.col0 + c0, v, RW);
          }
          if (ct == 0) g.counters[w.pt] = 0u;
        }
      }
      return true;
    };

    // Per-source state and one conversion step (A-ring position cur, unit w).
    // NF4: the 16 levels in registers (or this lane's copy of the pair table); block
    // constants fetched one step ahead.
    const uint32_t lut_tb =
        smem_u32(base + sp.lut) + (static_cast<uint32_t>(lane & (g.lut > 0 ? g.lut - 1 : 0)) << 2);
    const uint32_t lut_sh = g.lut == 16 ? 6u : 7u;  // bytes per table entry row: 4 x copies
    float lv[16];
    float mu = 0.f;
    const int slot = TMA_A ? lrow : t;  // A row slot (in TMEM: the lane this warp may access)
    int64_t bnext = 0;
    bool rowok = false, vnext = false;
    uint32_t cnext = 0;
    float snext = 0.f;
    int64_t bstep = 0;
    int cn = 0;  // MN-major: contraction index (weight row) of the next step's block
    // block index of this slot's first step in unit w
    auto first_block = [&](const Unit& w) -> int64_t {
      if (ASRC == A_NF4_K) {
        const int64_t n = w.row0 + slot;
        rowok = n < g.wN;
        return n * g.nbk + w.step0 + set;
      }
      const int kb = slot >> 6, nr = slot & 63;
      const int64_t kblk = w.row0 / 64 + kb;
      rowok = kblk < g.nbk;
      cn = (w.step0 + set) * kStep + nr;
      return (static_cast<int64_t>(w.step0 + set) * kStep + nr) * g.nbk + kblk;
    };
    // constants of this set's first step in unit un (none past the last unit)
    auto prefetch_unit = [&](int un) {
      vnext = false;
      if (un < g.nunits) {
        const Unit wn = unit_of(g, un);
        bnext = first_block(wn);
        vnext = rowok && set < wn.nst && (ASRC == A_NF4_K || cn < g.wN);
      }
      if (vnext && !in_bounds(bnext < g.cst_elems, 27)) vnext = false;
      if (vnext) {
        if (ASRC == A_CHANQ_MN) {
          snext = __ldg(g.cq_absmax + bnext);  // the group's absmax is its constant
        } else {
          cnext = g.code2[bnext];
          snext = __ldg(g.scale2 + (bnext >> 8));
        }
      }
    };
    // per-channel: the row's 2^b mapping values (unused entries 0), codes widened
    // to the 4-bit layout so the NF4 register lookup applies
    int cbits = 1;
    const uint8_t* prow = nullptr;
    bool cvalid = false;
    int64_t crow = 0;
    float mp[16];
    const uint32_t* s_t1 = reinterpret_cast<const uint32_t*>(base + sp.cq);  // 1-bit byte -> nibble word

    if constexpr (ASRC == A_NF4_K || ASRC == A_NF4_MN) {
#pragma unroll
      for (int kq = 0; kq < 16; ++kq) lv[kq] = s_lv[kq];
      mu = *g.mean;
      bstep = (ASRC == A_NF4_K) ? static_cast<int64_t>(NSET)
                                : static_cast<int64_t>(NSET) * kStep * g.nbk;
      prefetch_unit(u0);
    } else if constexpr (ASRC == A_CHANQ_MN) {
      bstep = static_cast<int64_t>(NSET) * kStep * g.nbk;
      prefetch_unit(u0);
    } else if constexpr (ASRC == A_CHANQ_K) {
      if (set == 0) {
        uint32_t* t1 = reinterpret_cast<uint32_t*>(base + sp.cq);
        for (int e = t; e < 256; e += 128) {
          uint32_t word = 0;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t hi = (static_cast<uint32_t>(e) >> (7 - 2 * m)) & 1u;
            const uint32_t lo = (static_cast<uint32_t>(e) >> (6 - 2 * m)) & 1u;
            word |= ((hi << 4) | lo) << (8 * m);
          }
          t1[e] = word;
        }
      }
      named_sync(2, NCONV);  // the table is read by every converter set
    }

    // Hand a finished A stage to the MMA.
    auto publish = [&](const ConvCursor& cur, const uint32_t (&o)[32]) {
      if (TMA_A) {
        tc_fence_after();
        tmem_st32(tmem + (static_cast<uint32_t>(q * 32) << 16) + a_col + 32u * cur.s2, o);
        tmem_wait_st();
        tc_fence_before();
      } else {
        store_row_sw128(base + sp.ring2 + cur.s2 * sp.slot2, slot, o);
        fence_proxy_async();
      }
      mbar_arrive(&full2[cur.s2]);
    };
    // Wait until step cur's packed data has landed and its A stage is free (the MMA
    // of the position S2 earlier has completed).
    auto acquire = [&](const ConvCursor& cur, unsigned int site) -> bool {
      if (!wait_or_abort(&full1[cur.s], cur.ph, g.wait_ns, &s_abort, site)) return false;
      if (cur.r >= S2 && !wait_or_abort(&empty1[cur.sj], cur.phj, g.wait_ns, &s_abort, site + 1))
        return false;
      return true;
    };
    // The adapter position writes no A stage, but its full2 arrival must fall in that
    // stage's next phase: wait for the stage's previous user as a conversion would.
    auto pass_ext = [&](const ConvCursor& cur) -> bool {
      if (cur.r >= S2 && !wait_or_abort(&empty1[cur.sj], cur.phj, g.wait_ns, &s_abort, 35))
        return false;
      mbar_arrive(&full2[cur.s2]);
      return true;
    };

    // One conversion step; false when a wait gave up.
    auto step = [&](const Unit& w, const ConvCursor& cur, int u) -> bool {
      if constexpr (ASRC == A_NF4_K || ASRC == A_NF4_MN || ASRC == A_CHANQ_MN) {
        const bool valid = vnext;
        const float ch = !valid ? 0.f
                         : (ASRC == A_CHANQ_MN ? snext
                                               : fmaf(e4m3_to_f32(static_cast<uint8_t>(cnext)), snext, mu));
        // constants of this set's next step: in this unit, else in the CTA's next unit
        if (cur.i + NSET < w.nst) {
          bnext += bstep;
          cn += NSET * kStep;
          vnext = rowok && (ASRC == A_NF4_K || cn < g.wN);
          if (vnext && !in_bounds(bnext < g.cst_elems, 27)) vnext = false;
          if (vnext) {
            if (ASRC == A_CHANQ_MN) {
              snext = __ldg(g.cq_absmax + bnext);
            } else {
              cnext = g.code2[bnext];
              snext = __ldg(g.scale2 + (bnext >> 8));
            }
          }
        } else {
          prefetch_unit(u + ustep);
        }
        if (!acquire(cur, 31)) return false;
        const uint8_t* pk = base + cur.s * sp.slot1 + sp.off_p1;
        const uint8_t* src =
            (ASRC == A_NF4_K) ? pk + slot * 32 : pk + (slot & 63) * 64 + (slot >> 6) * 32;
        uint32_t o[32];
        if constexpr (ASRC == A_CHANQ_MN) {
          // this step's contraction row (slot & 63): its 16 mapping values from the
          // table tile that came with the codes (unused entries 0)
          const float4* tb = reinterpret_cast<const float4*>(base + cur.s * sp.slot1 + sp.off_t1 +
                                                             (slot & 63) * 64);
          float tv[16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 f = tb[q4];
            tv[4 * q4] = f.x; tv[4 * q4 + 1] = f.y; tv[4 * q4 + 2] = f.z; tv[4 * q4 + 3] = f.w;
          }
          nf4_block_to_bf16(src, ch, tv, o);
        } else if (g.lut) {
          nf4_block_lut(src, pack_bf16x2(ch, ch), lut_tb, lut_sh, o);
        } else {
          nf4_block_to_bf16(src, ch, lv, o);
        }
        publish(cur, o);
      } else if constexpr (ASRC == A_CHANQ_K) {
        const int gi = w.step0 + cur.i;
        // the group's codes and scale (issued before the waits)
        uint32_t cw[8];
        float gm = 0.f;
        if (cvalid) {
          gm = __ldg(g.cq_absmax + crow * g.nbk + gi);
          // A row holds K b / 8 bytes (a multiple of 8, not of 16, e.g. K = 448) and a
          // group 8 b bytes, so only 8-byte loads are aligned for every shape.
          const uint2* src = reinterpret_cast<const uint2*>(prow + static_cast<int64_t>(gi) * 8 * cbits);
          if (cbits == 4) {
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              const uint2 a = __ldg(src + kq);
              cw[2 * kq] = a.x;
              cw[2 * kq + 1] = a.y;
            }
          } else if (cbits == 2) {
            const uint2 a0 = __ldg(src), a1 = __ldg(src + 1);
            const uint32_t in[4] = {a0.x, a0.y, a1.x, a1.y};
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              // byte x = c0 c1 c2 c3 (2 bits each, first at the top) -> (c0 c1), (c2 c3)
              const uint32_t x = in[kq];
              const uint32_t hi = ((x >> 2) & 0x30303030u) | ((x >> 4) & 0x03030303u);
              const uint32_t lo = ((x << 2) & 0x30303030u) | (x & 0x03030303u);
              cw[2 * kq] = __byte_perm(hi, lo, 0x5140);
              cw[2 * kq + 1] = __byte_perm(hi, lo, 0x7362);
            }
          } else {
            const uint2 a = __ldg(src);
#pragma unroll
            for (int kq = 0; kq < 8; ++kq) cw[kq] = s_t1[((kq < 4 ? a.x : a.y) >> (8 * (kq & 3))) & 0xFFu];
          }
        } else {
#pragma unroll
          for (int kq = 0; kq < 8; ++kq) cw[kq] = 0u;
        }
        if (!acquire(cur, 33)) return false;
        uint32_t o[32];
        Nf4Planes P;
        nf4_planes(mp, gm, P);
#pragma unroll
        for (int kq = 0; kq < 8; ++kq) nf4_lookup8(cw[kq], P, &o[4 * kq]);
        publish(cur, o);
      }
      return true;
    };
    // per-unit state of the per-channel source: this row's bits, codes and mapping
    auto unit_rows = [&](const Unit& w) {
      if constexpr (ASRC == A_CHANQ_K) {
        crow = w.row0 + slot;
        cvalid = crow < g.wN;
        int64_t mo = 0;
        cbits = 1;
        if (cvalid) {
          cbits = g.cq_bits[crow];
          prow = g.cq_packed + g.cq_row_off[crow];
          mo = g.cq_map_off[crow];
        }
        const int nmap = cvalid ? (1 << cbits) : 0;
#pragma unroll
        for (int c = 0; c < 16; ++c) mp[c] = c < nmap ? g.cq_map[mo + c] : 0.f;
      }
    };

    // The unit loop. Each set converts its first step of unit k before the epilogue
    // of unit k-1 (those steps wait only for MMAs of earlier units), so the MMA has
    // work the moment the accumulator is free again.
    const int ahead = min(NSET, S2);
    int rbase = 0;  // ring position of the unit's first step
    int up = -1;    // the previous unit, while its epilogue is still due
    // One pass per unit of this CTA and a last one for the final epilogue; the
    // epilogue and the adapter write each have a single call site (smaller code).
    for (int k = 0;; ++k) {
      const int u = u0 + k * ustep;
      const bool live = u < g.nunits;  // a unit to convert (else only the last epilogue)
      // (dense sources have no A ring: the cursor gets a dummy depth)
      ConvCursor cur(set, rbase, S1, DEQ ? S2 : 1);
      if (live) {
        const Unit w = unit_of(g, u);
        unit_rows(w);
        if constexpr (ASRC == A_NF4_K || ASRC == A_NF4_MN || ASRC == A_CHANQ_MN) {
          if (set >= w.nst) prefetch_unit(u + ustep);  // no step of this set here
        }
        // positions converted before the previous unit's epilogue
        if (DEQ && up >= 0 && !dead) {
          const int pre = min(ahead, w.nst + (w.ext ? 1 : 0));
          for (; cur.i < pre; cur.next(NSET, S1, S2)) {
            if (!(cur.i < w.nst ? step(w, cur, u) : pass_ext(cur))) {
              dead = true;
              break;
            }
          }
        }
      }
      if (up >= 0) {
        const bool more = epilogue(up, k - 1);
        up = -1;
        if (!more) break;
      }
      if (!live) break;
      const Unit w = unit_of(g, u);  // recomputed: not kept live across the epilogue
      const int nload = w.nst + (w.ext ? 1 : 0);
      if (w.ext && set == 0) write_ext(w);
      if (DEQ && !dead) {
        for (; cur.i < w.nst; cur.next(NSET, S1, S2)) {
          if (!step(w, cur, u)) {
            dead = true;
            break;
          }
        }
        // the adapter position, when it falls to this set
        if (!dead && cur.i == w.nst && w.ext && !pass_ext(cur)) dead = true;
      }
      up = u;
      rbase += nload;
    }
    if (g.stage && t == 0) bulk_wait0();  // the output stores have completed
    tc_fence_before();
  }

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
