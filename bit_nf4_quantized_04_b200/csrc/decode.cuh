// Forward of the NF4 linear layer for a handful of tokens (M <= 16), the decode case
// of "QLoRA: Efficient Finetuning of Quantized LLMs" (Heng's Blog, 贡献一/贡献二 and the
// dequantize-then-multiply forward): h = x bf16(W_hat)^T + s (x A^T) B^T.
//
// With M <= 16 the layer streams 4.127 bits per weight and does 2 M flops per weight,
// so it is bound by HBM and by the dequantization, not by the tensor cores. Each warp
// owns a contiguous run of (8-row tile, 256-column group) items and streams their
// packed codes through its own ring of shared-memory slots (cp.async, kDecRing items
// in flight). Lane (g, t) dequantizes row g of the tile, block t of the group, in
// registers (the exact per-block product table of the prefill path, looked up with
// byte permutes), and the results are the B operand of mma.sync.m16n8k16, with x (the
// 16-row A operand, tokens past M as zeros) staged once per CTA in shared memory.
// Nothing passes through TMEM or an mbarrier pipeline.
//
// K is permuted inside each 256-column group so that lane t of a quad holds the 64
// columns of block t: a lane dequantizes one whole NF4 block with one product table,
// and x is read with the same permutation (a sum over K does not depend on the order
// of its terms). A warp writes the partial tile of every tile it touches to a
// workspace as it goes; after its run it counts itself in for those tiles, and the
// last warp to arrive at a tile adds the partial tiles in a fixed order, adds the
// adapter term and writes bf16. A cluster of kDecPrepCtas CTAs, launched just before
// on SMs the main grid leaves free, computes x A^T and clears the tile counters; the
// main kernel waits for it (programmatic dependent launch) only after its run.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "gemm.cuh"

namespace qnf4 {

constexpr int kDecWarps = 24;                  // warps per CTA of the main kernel (one CTA per SM)
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecRows = 8;                    // weight rows per tile (the MMA's N)
constexpr int kDecMaxTok = 16;                 // tokens handled by this path (the MMA's M)
constexpr int kDecMaxChunks = 8;               // K chunks (x staging windows)
constexpr int kDecSmem = 64 * 1024;            // x window per CTA (M rows)
constexpr int kDecRing = 4;                    // items in flight per warp
constexpr int kDecItemBytes = 1024;            // codes of one item: 8 rows x 128 bytes
constexpr int kDecRingBytes = kDecWarps * kDecRing * kDecItemBytes;
constexpr int kDecMaxFin = 8;                  // tiles a warp hands over after its run (at most)
constexpr int kDecSlot = 128;                  // floats of a partial tile (16 tokens x 8 rows)
constexpr int kDecPrepCtas = 8;                // the prep kernel: one cluster
constexpr int kDecPrepThreads = 512;
constexpr int kDecPrepWarps = kDecPrepThreads / 32;
constexpr int kDecULd = 64;                    // row stride (elements) of x A^T
constexpr int kDecUShare = kDecMaxTok * kDecULd;  // floats of x A^T (16 tokens x 64)

struct DecArgs {
  const uint8_t* packed;   // [N, K/2] codes, element 2j in the high nibble of byte j
  const uint8_t* code2;    // [N K / 64] E4M3 codes of the block constants
  const float* scale2;     // [ceil(N K / 64 / 256)]
  const float* mean;       // [1]
  const uint16_t* x;       // [M, K] bf16
  const uint16_t* A;       // [r, K] bf16
  const uint16_t* B;       // [N, r] bf16
  const float* u;          // [16, 64] fp32 x A^T, zero past M and r (k_dec_prep)
  uint16_t* h;             // [M, N] bf16
  float* part;             // [T, nchunks, jmax, kDecSlot] fp32 partial tiles
  unsigned int* cnt;       // [T] arrivals per tile (zeroed by k_dec_prep)
  int64_t N, K;
  int64_t T;               // 8-row tiles
  int M, r, KB, jmax, nchunks;
  float scale;             // s
  int xrows;                   // rows of the x window: M, plus one row of zeros if M < 16
  int gb[kDecMaxChunks + 1];   // first 256-column group of each chunk
  int cb[kDecMaxChunks + 1];   // first CTA of each chunk
  float levels[16];
};

// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
QNF4_DEV void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
QNF4_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
QNF4_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

QNF4_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

QNF4_DEV uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// a 32-bit pair of bf16 at p (4-byte aligned) or zero
QNF4_DEV uint32_t ld_pair(const uint16_t* p, bool ok) {
  return ok ? __ldg(reinterpret_cast<const unsigned int*>(p)) : 0u;
}

// nf4_lookup8 with its three right shifts done as high-half multiplies (the integer
// multiply-add pipe) instead of shifts, leaving the logic pipe the 16 byte permutes
// and three masks: the same 8 codes -> 4 bf16 pairs.
QNF4_DEV void nf4_lookup8_m(uint32_t w, const Nf4Planes& P, uint32_t* o) {
  const uint32_t sa = w & 0x77777777u;
  const uint32_t sb = __umulhi(sa, 0x10000u);                          // sa >> 16
  const uint32_t ta = (__umulhi(w, 0x80000000u) & 0x4444u) | 0x3210u;  // (w >> 1) ...
  const uint32_t tb = (__umulhi(w, 0x8000u) & 0x4444u) | 0x3210u;      // (w >> 17) ...
  const uint32_t la = __byte_perm(__byte_perm(P.l[0], P.l[1], sa), __byte_perm(P.l[2], P.l[3], sa), ta);
  const uint32_t ha = __byte_perm(__byte_perm(P.h[0], P.h[1], sa), __byte_perm(P.h[2], P.h[3], sa), ta);
  const uint32_t lb = __byte_perm(__byte_perm(P.l[0], P.l[1], sb), __byte_perm(P.l[2], P.l[3], sb), tb);
  const uint32_t hb = __byte_perm(__byte_perm(P.h[0], P.h[1], sb), __byte_perm(P.h[2], P.h[3], sb), tb);
  o[0] = __byte_perm(la, ha, 0x4051);
  o[1] = __byte_perm(la, ha, 0x6273);
  o[2] = __byte_perm(lb, hb, 0x4051);
  o[3] = __byte_perm(lb, hb, 0x6273);
}

QNF4_DEV void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// floor(n / d) for 0 <= n < 2^53, 0 < d: the quotient of the two doubles is within
// n 2^-53 of n / d, less than the gap 1/d to the next integer below when n / d is not
// an integer, and exact when it is; so the floor is exact (the plan checks the bound).
__host__ __device__ inline int64_t dec_div(int64_t n, int64_t d) {
  return static_cast<int64_t>(floor(static_cast<double>(n) / static_cast<double>(d)));
}

// Work split of one chunk: its items (tile p, group q) are numbered p * gc + q and
// warp w of the chunk's tw warps takes [w items / tw, (w + 1) items / tw).
struct DecSplit {
  int64_t items, tw;
  int gc;
  __host__ __device__ int64_t begin(int64_t w) const { return dec_div(w * items, tw); }
  // the warp whose run holds item i (the largest w with begin(w) <= i)
  __host__ __device__ int64_t owner(int64_t i) const { return dec_div((i + 1) * tw + items - 1, items) - 1; }
  __host__ __device__ int ncon(int64_t p) const {
    return static_cast<int>(owner(p * gc + gc - 1) - owner(p * gc) + 1);
  }
};

__host__ __device__ inline DecSplit dec_split(int64_t T, int gb0, int gb1, int ctas) {
  DecSplit s;
  s.gc = gb1 - gb0;
  s.items = T * s.gc;
  s.tw = s.items < static_cast<int64_t>(ctas) * kDecWarps ? s.items
                                                          : static_cast<int64_t>(ctas) * kDecWarps;
  return s;
}

// A lane's stream over the items of a warp's run in one chunk (item = tile p, group q
// of the chunk): its row r = 8 p + g, its block b = 4 (g0 + q) + t, the byte offset of
// the 32-byte block row in the packed codes, the index of the block constant and the
// groups left in the current tile. A step is a few adds (32-bit: the plan keeps
// N K / 2 below 2^31).
struct DecStream {
  uint32_t off, ci;
  int row, blk, left, p;
  QNF4_DEV void init(const DecArgs& a, int p0, int q0, int g0, int gc, int gq, int tq) {
    p = p0;
    row = p0 * kDecRows + gq;
    blk = 4 * (g0 + q0) + tq;
    left = gc - q0;
    off = static_cast<uint32_t>(row) * static_cast<uint32_t>(a.K / 2) + static_cast<uint32_t>(blk) * 32u;
    ci = static_cast<uint32_t>(row) * static_cast<uint32_t>(a.KB) + static_cast<uint32_t>(blk);
  }
  // jumps at the end of a tile: 8 rows down, back to the chunk's first group
  QNF4_DEV void step(int gc, uint32_t off_jump, uint32_t ci_jump) {
    if (--left == 0) {
      left = gc;
      ++p;
      row += kDecRows;
      blk -= 4 * (gc - 1);
      off += off_jump;
      ci += ci_jump;
    } else {
      blk += 4;
      off += 128u;
      ci += 4u;
    }
  }
  // the lane's row and block exist (rows past N and blocks past K read as zeros)
  QNF4_DEV bool valid(const DecArgs& a) const { return blk < a.KB && row < a.N; }
};

// The block constant of one item for this lane: E4M3 code and second-level scale.
struct DecConst {
  uint32_t e;
  float s;
};

QNF4_DEV void dec_consts(const DecArgs& a, const DecStream& st, DecConst& k) {
  const bool v = st.valid(a);
  k.e = v ? __ldg(a.code2 + st.ci) : 0u;
  k.s = v ? __ldg(a.scale2 + (st.ci >> 8)) : 0.f;
}

// Ring slot layout: this lane's 16-byte half k of its 32-byte block row sits at slot
// + (32 k + lane) 16, so a warp's copies and reads of one half are 512 consecutive
// bytes.
QNF4_DEV void dec_fetch(const DecArgs& a, uint32_t slot, const DecStream& st, int lane) {
  const bool v = st.valid(a);
  const uint8_t* src = v ? a.packed + st.off : a.packed;
  const uint32_t n = v ? 16u : 0u;
  cp_async16(slot + lane * 16, src, n);
  cp_async16(slot + (32 + lane) * 16, v ? src + 16 : src, n);
}

// The number of warps, over all chunks, whose runs touch tile p.
QNF4_DEV int dec_expect(const DecArgs& a, int64_t p) {
  int e = 0;
  for (int c = 0; c < a.nchunks; ++c) e += dec_split(a.T, a.gb[c], a.gb[c + 1], a.cb[c + 1] - a.cb[c]).ncon(p);
  return e;
}

// x window layout in shared memory: 16-byte chunk j (8 columns) of block bl of row
// `row` sits at ((row nb + bl) 8 + (j ^ swz)) 16 with swz = ((row & 1) << 2) | (bl & 3),
// so the 8 lanes of a quarter warp (two tokens times four blocks) hit 8 distinct
// 16-byte bank groups. The staging writes every swizzle of every row, so the tokens
// past M, which read the zero row with their own swizzle, find zeros too.
QNF4_DEV uint32_t dec_xoff(int row, int bl, int j, int nb) {
  const int swz = ((row & 1) << 2) | (bl & 3);
  return static_cast<uint32_t>(((row * nb + bl) * 8 + (j ^ swz)) * 16);
}

QNF4_DEV float* dec_slot(const DecArgs& a, int64_t p, int c, int j) {
  return a.part + ((p * a.nchunks + c) * a.jmax + j) * kDecSlot;
}

// The last contributor of tile p adds the partial tiles in (chunk, contributor)
// order, adds the adapter term s (x A^T) B_tile^T as m16n8k16 products (A fragments
// ub = bf16(s x A^T) for tokens g, g + 8; B fragments from row g of the tile's B
// rows; both zero past M, N and r) and writes the bf16 tile. acc holds tokens
// (g, g + 8) x rows (2 t, 2 t + 1) of the tile.
QNF4_DEV void dec_finish(const DecArgs& a, int64_t p, int gq, int tq, int lane) {
  uint32_t la[4][4], lb[4][2];
  const int64_t nrow = p * kDecRows + gq;
  const bool vr = nrow < a.N;
  const uint16_t* brow = a.B + nrow * a.r;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int j = 16 * s + 2 * tq;
    const bool sv = 16 * s < a.r;
    const float* u0 = a.u + gq * kDecULd + j;
    const float* u1 = a.u + (gq + 8) * kDecULd + j;
    const float2 v00 = sv ? __ldcg(reinterpret_cast<const float2*>(u0)) : make_float2(0.f, 0.f);
    const float2 v01 = sv ? __ldcg(reinterpret_cast<const float2*>(u0 + 8)) : make_float2(0.f, 0.f);
    const float2 v10 = sv ? __ldcg(reinterpret_cast<const float2*>(u1)) : make_float2(0.f, 0.f);
    const float2 v11 = sv ? __ldcg(reinterpret_cast<const float2*>(u1 + 8)) : make_float2(0.f, 0.f);
    la[s][0] = pack_bf16x2(v00.x * a.scale, v00.y * a.scale);  // token g,     columns j, j+1
    la[s][1] = pack_bf16x2(v10.x * a.scale, v10.y * a.scale);  // token g + 8, columns j, j+1
    la[s][2] = pack_bf16x2(v01.x * a.scale, v01.y * a.scale);  // token g,     columns j+8, j+9
    la[s][3] = pack_bf16x2(v11.x * a.scale, v11.y * a.scale);  // token g + 8, columns j+8, j+9
    uint32_t e[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int jj = j + (v & 1) + 8 * (v >> 1);
      e[v] = (sv && vr && jj < a.r) ? static_cast<uint32_t>(__ldg(brow + jj)) : 0u;
    }
    lb[s][0] = e[0] | (e[1] << 16);  // row g, columns j, j+1
    lb[s][1] = e[2] | (e[3] << 16);  // row g, columns j+8, j+9
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  // lane c < nchunks counts chunk c's contributors
  const int nl = lane < a.nchunks ? dec_split(a.T, a.gb[lane], a.gb[lane + 1], a.cb[lane + 1] - a.cb[lane]).ncon(p) : 0;
  for (int cc = 0; cc < a.nchunks; ++cc) {
    const int n = __shfl_sync(0xffffffffu, nl, cc);
    const float4* base = reinterpret_cast<const float4*>(dec_slot(a, p, cc, 0));
    for (int jj = 0; jj < n; jj += 4) {
      float4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[k] = jj + k < n ? __ldcg(base + (jj + k) * (kDecSlot / 4) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[0] += v[k].x;
        acc[1] += v[k].y;
        acc[2] += v[k].z;
        acc[3] += v[k].w;
      }
    }
  }
#pragma unroll
  for (int s = 0; s < 4; ++s)
    if (16 * s < a.r) mma_16816(acc, la[s][0], la[s][1], la[s][2], la[s][3], lb[s][0], lb[s][1]);
  const int64_t n0 = p * kDecRows + 2 * tq;
  const int t0 = gq, t1 = gq + 8;
  if (t0 < a.M && n0 < a.N) a.h[t0 * a.N + n0] = f2bf(acc[0]);
  if (t0 < a.M && n0 + 1 < a.N) a.h[t0 * a.N + n0 + 1] = f2bf(acc[1]);
  if (t1 < a.M && n0 < a.N) a.h[t1 * a.N + n0] = f2bf(acc[2]);
  if (t1 < a.M && n0 + 1 < a.N) a.h[t1 * a.N + n0 + 1] = f2bf(acc[3]);
}

// Counts this warp in for the n parked tiles p0, p0 + 1, ... (their partial tiles are
// in their slots; the counters are the prep kernel's; lane f holds the contributor
// count of tile p0 + f): all arrivals go out before any answer is awaited; then the
// warp finishes the tiles it arrived last at.
QNF4_DEV void dec_count_in(const DecArgs& a, int p0, int n, int expect_l, int gq, int tq, int lane) {
  int fin[kDecMaxFin], expect[kDecMaxFin];
  unsigned int old[kDecMaxFin];
#pragma unroll
  for (int f = 0; f < kDecMaxFin; ++f) {
    fin[f] = p0 + f;
    expect[f] = __shfl_sync(0xffffffffu, expect_l, f);
    if (f >= n) expect[f] = 0;
  }
#pragma unroll
  for (int f = 0; f < kDecMaxFin; ++f) {
    old[f] = 0u;
    if (lane == 0 && expect[f] > 1) old[f] = atomicAdd(a.cnt + fin[f], 1u);
  }
  bool any = false;
  bool mine[kDecMaxFin];
#pragma unroll
  for (int f = 0; f < kDecMaxFin; ++f) {
    old[f] = __shfl_sync(0xffffffffu, old[f], 0);
    mine[f] = f < n && (expect[f] == 1 || static_cast<int>(old[f]) == expect[f] - 1);
    any |= mine[f];
  }
  if (!any) return;
  __threadfence();
#pragma unroll
  for (int f = 0; f < kDecMaxFin; ++f)
    if (mine[f]) dec_finish(a, fin[f], gq, tq, lane);
}

// One warp's run of items in chunk c. See the file comment for the data layout. TWO:
// tokens 8..15 exist (M > 8), so x has a second 8-row half.
template <bool TWO>
__global__ void __launch_bounds__(kDecThreads, 1) k_dec(const __grid_constant__ DecArgs a) {
  extern __shared__ __align__(128) uint8_t dsm[];
  griddep_launch_dependents();
  int c = 0;
  while (c + 1 < a.nchunks && static_cast<int>(blockIdx.x) >= a.cb[c + 1]) ++c;
  const int g0 = a.gb[c], g1 = a.gb[c + 1];
  const DecSplit sp = dec_split(a.T, g0, g1, a.cb[c + 1] - a.cb[c]);
  const int gc = sp.gc;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int w = static_cast<int>(blockIdx.x - a.cb[c]) * kDecWarps + warp;
  const bool active = w < sp.tw;
  const int ib = active ? static_cast<int>(sp.begin(w)) : 0;  // items < 2^26 (the plan)
  const int ie = active ? static_cast<int>(sp.begin(w + 1)) : 0;

  const uint32_t ring = smem_u32(dsm) + warp * (kDecRing * kDecItemBytes);
  // the x window, 128-byte aligned (the launch adds 128 bytes of slack)
  const uint32_t xs0 = (smem_u32(dsm) + kDecRingBytes + 127u) & ~127u;

  // ---- stage x[:M, 256 g0 : 256 g1] (columns past K as zeros, and a row of zeros
  // that the tokens past M read): the oldest copy group of every thread
  const int nb = 4 * (g1 - g0);  // 64-column blocks in the window
  const int kb0 = 4 * g0;
  {
    // thread i copies 16-byte chunk j = i % 8 of the (row, block) pairs i / 8, i / 8 +
    // kDecThreads / 8, ... (row-major)
    const int j = threadIdx.x & 7;
    int e = threadIdx.x >> 3;
    int row = e / nb, bl = e - (e / nb) * nb;
    for (; row < a.xrows; e += kDecThreads / 8) {
      const bool in = row < a.M && kb0 + bl < a.KB;
      const uint16_t* src = in ? a.x + static_cast<int64_t>(row) * a.K + static_cast<int64_t>(kb0 + bl) * 64 + j * 8 : a.x;
      cp_async16(xs0 + dec_xoff(row, bl, j, nb), src, in ? 16u : 0u);
      bl += kDecThreads / 8;
      while (bl >= nb) {
        bl -= nb;
        ++row;
      }
    }
  }
  cp_async_commit();

  // ---- streams: the item being computed, its constants one ahead, copies kDecRing ahead
  const int p0 = ib / gc;
  const int q0 = ib - p0 * gc;
  const uint32_t off_jump = static_cast<uint32_t>(4 * a.K) - 128u * static_cast<uint32_t>(gc - 1);
  const uint32_t ci_jump = static_cast<uint32_t>(kDecRows * a.KB) - 4u * static_cast<uint32_t>(gc - 1);
  DecStream sc, sk, sf;
  sc.init(a, p0, q0, g0, gc, gq, tq);
  sf = sc;
#pragma unroll
  for (int d = 0; d < kDecRing; ++d) {
    if (ib + d < ie) dec_fetch(a, ring + d * kDecItemBytes, sf, lane);
    cp_async_commit();
    sf.step(gc, off_jump, ci_jump);
  }
  // the block constants of the whole run into L2 (lane l < 8: row l of each tile)
  if (lane < kDecRows && ib < ie) {
    for (int pp = p0; pp * gc < ie; ++pp) {
      const int64_t row = static_cast<int64_t>(pp) * kDecRows + lane;
      if (row >= a.N) continue;
      const int qlo = pp == p0 ? q0 : 0;
      const int qhi = min(gc, ie - pp * gc) - 1;
      const int64_t i0 = row * a.KB + 4 * (g0 + qlo), i1 = row * a.KB + min(a.KB - 1, 4 * (g0 + qhi) + 3);
      prefetch_l2(a.code2 + i0);
      prefetch_l2(a.code2 + i1);
      prefetch_l2(a.scale2 + (i0 >> 8));
      prefetch_l2(a.scale2 + (i1 >> 8));
    }
  }
  DecConst cur;
  if (ib < ie) dec_consts(a, sc, cur);
  sk = sc;
  sk.step(gc, off_jump, ci_jump);
  cp_async_wait<kDecRing - 1>();  // the x window and the first item
  __syncthreads();
  if (!active) return;

  // this lane's x rows (tokens g and g + 8, or the zero row); the 16-byte chunk j of
  // block bl of a row lies at (row, block bl) ^ (16 swz) ^ (16 j), swz the token's
  // swizzle (the same for g and g + 8)
  const uint32_t swz16 = static_cast<uint32_t>(((gq & 1) << 2) | tq) << 4;
  const uint32_t xr0 = (xs0 + static_cast<uint32_t>((gq < a.M ? gq : a.M) * nb) * 128u - kb0 * 128u);
  const uint32_t xr1 = (xs0 + static_cast<uint32_t>((gq + 8 < a.M ? gq + 8 : a.M) * nb) * 128u - kb0 * 128u);
  // slot of this warp's partial tiles: only its first tile can have earlier contributors
  const int j_first = static_cast<int>(w - sp.owner(static_cast<int64_t>(p0) * gc));
  // the run's tiles are p0, p0 + 1, ... (at most kDecMaxFin, by the plan); lane f counts
  // the contributors of tile p0 + f
  const int ntiles = ib < ie ? (ie - 1) / gc - p0 + 1 : 0;
  const int expect_l = lane < ntiles ? dec_expect(a, p0 + lane) : 0;

  const float mu = __ldg(a.mean);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t slot = ring;
  const uint32_t ring_end = ring + kDecRing * kDecItemBytes;

  for (int i = ib; i < ie; ++i) {
    DecConst nxt;
    if (i + 1 < ie) dec_consts(a, sk, nxt);

    // ---- dequantize this item and multiply
    {
      const uint4 c0 = lds_u4(slot + lane * 16), c1 = lds_u4(slot + (32 + lane) * 16);
      const uint32_t blo = static_cast<uint32_t>(sc.blk) * 128u;  // (block - kb0) 128 + kb0 128
      const uint32_t xb0 = (xr0 + blo) ^ swz16, xb1 = (xr1 + blo) ^ swz16;
      Nf4Planes P;
      nf4_planes(a.levels, fmaf(e4m3_to_f32(static_cast<uint8_t>(cur.e)), cur.s, mu), P);
      const uint32_t wd[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t o[4];
        nf4_lookup8_m(wd[j], P, o);
        const uint4 x0 = lds_u4(xb0 ^ static_cast<uint32_t>(j << 4));
        if (TWO) {
          const uint4 x1 = lds_u4(xb1 ^ static_cast<uint32_t>(j << 4));
          mma_16816(acc, x0.x, x1.x, x0.y, x1.y, o[0], o[1]);
          mma_16816(acc, x0.z, x1.z, x0.w, x1.w, o[2], o[3]);
        } else {
          // columns 8 j .. 8 j + 7 of block t: two k16 slices of the permuted K
          mma_16816(acc, x0.x, 0u, x0.y, 0u, o[0], o[1]);
          mma_16816(acc, x0.z, 0u, x0.w, 0u, o[2], o[3]);
        }
      }
    }
    // ---- refill the slot (its codes are in registers now) with the item kDecRing ahead
    if (i + kDecRing < ie) dec_fetch(a, slot, sf, lane);
    cp_async_commit();
    sf.step(gc, off_jump, ci_jump);
    slot += kDecItemBytes;
    if (slot == ring_end) slot = ring;

    // ---- end of this warp's part of tile p: park the partial tile
    if (i + 1 == ie || sc.left == 1) {
      const int j = sc.p == p0 ? j_first : 0;
      __stcg(reinterpret_cast<float4*>(dec_slot(a, sc.p, c, j)) + lane,
             make_float4(acc[0], acc[1], acc[2], acc[3]));
      acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    }
    cur = nxt;
    sc.step(gc, off_jump, ci_jump);
    sk.step(gc, off_jump, ci_jump);
    cp_async_wait<kDecRing - 1>();  // the next item has landed
  }

  // ---- after the run: count in for the parked tiles (the prep kernel has cleared the
  // counters and written x A^T by now)
  griddep_wait();
  __threadfence();  // the partial tiles before the arrivals
  __syncwarp();
  if (ntiles > kDecMaxFin) set_err(61);  // the plan bounds the tiles of a run
  dec_count_in(a, p0, min(ntiles, kDecMaxFin), expect_l, gq, tq, lane);
}

// The prep kernel of the decode forward, one cluster of kDecPrepCtas CTAs:
// (1) clears the main kernel's tile counters;
// (2) computes x A^T in fp32 (16 x 64, zero past M and r): CTA k takes a contiguous
//     share of the 64-column blocks of K, its warp w the 16-column slices w,
//     w + kDecPrepWarps, ... of that share, four slices' fragments loaded at a time and
//     multiplied with mma.sync (x as the 16-row A operand, A^T as up to eight 8-column
//     B tiles); the warps' sums are added in warp order, then the CTAs' in rank order
//     (CTA k adding outputs k, k + kDecPrepCtas, ... from the others' shared memory).
__global__ void __launch_bounds__(kDecPrepThreads) k_dec_prep(const uint16_t* __restrict__ x,
                                                              const uint16_t* __restrict__ A,
                                                              int M, int64_t K, int r,
                                                              float* __restrict__ u,
                                                              unsigned int* __restrict__ cnt,
                                                              int64_t T) {
  namespace cg = cooperative_groups;
  extern __shared__ float s_red[];  // [kDecPrepWarps][kDecUShare]
  __shared__ float s_share[kDecUShare];
  cg::cluster_group cl = cg::this_cluster();
  griddep_wait();
  griddep_launch_dependents();
  const int rank = static_cast<int>(cl.block_rank());
  for (int64_t p = static_cast<int64_t>(rank) * kDecPrepThreads + threadIdx.x; p < T;
       p += static_cast<int64_t>(kDecPrepCtas) * kDecPrepThreads)
    cnt[p] = 0u;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t kb = K / 64, per = (kb + kDecPrepCtas - 1) / kDecPrepCtas;
  const int64_t k0 = min(kb, rank * per) * 64, k1 = min(kb, (rank + 1) * per) * 64;
  const bool t0ok = gq < M, t1ok = gq + 8 < M;
  const uint16_t* x0 = x + static_cast<int64_t>(t0ok ? gq : 0) * K;
  const uint16_t* x1 = x + static_cast<int64_t>(t1ok ? gq + 8 : 0) * K;
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  constexpr int kB = 4;  // slices per load batch
  for (int64_t s0 = k0 + 16 * warp; s0 < k1; s0 += 16 * kDecPrepWarps * kB) {
    uint32_t xa[kB][4], ab[kB][8][2];
#pragma unroll
    for (int v = 0; v < kB; ++v) {
      const int64_t ks = s0 + 16 * kDecPrepWarps * v;
      const bool in = ks < k1;
      const int64_t kk = (in ? ks : 0) + 2 * tq;
      xa[v][0] = ld_pair(x0 + kk, in && t0ok);
      xa[v][1] = ld_pair(x1 + kk, in && t1ok);
      xa[v][2] = ld_pair(x0 + kk + 8, in && t0ok);
      xa[v][3] = ld_pair(x1 + kk + 8, in && t1ok);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int j = 8 * nt + gq;
        const bool ok = in && 8 * nt < r && j < r;
        const uint16_t* ar = A + static_cast<int64_t>(ok ? j : 0) * K + kk;
        ab[v][nt][0] = ld_pair(ar, ok);
        ab[v][nt][1] = ld_pair(ar + 8, ok);
      }
    }
#pragma unroll
    for (int v = 0; v < kB; ++v)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        if (8 * nt < r)
          mma_16816(acc[nt], xa[v][0], xa[v][1], xa[v][2], xa[v][3], ab[v][nt][0], ab[v][nt][1]);
  }
  // acc[nt]: tokens (g, g + 8) x adapter columns (8 nt + 2 t, + 1)
  float* mine = s_red + warp * kDecUShare;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int j = 8 * nt + 2 * tq;
    mine[gq * kDecULd + j] = acc[nt][0];
    mine[gq * kDecULd + j + 1] = acc[nt][1];
    mine[(gq + 8) * kDecULd + j] = acc[nt][2];
    mine[(gq + 8) * kDecULd + j + 1] = acc[nt][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kDecUShare; i += kDecPrepThreads) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < kDecPrepWarps; ++k) t += s_red[k * kDecUShare + i];
    s_share[i] = t;
  }
  cl.sync();
  for (int i = rank + kDecPrepCtas * threadIdx.x; i < kDecUShare; i += kDecPrepCtas * kDecPrepThreads) {
    float v[kDecPrepCtas];
#pragma unroll
    for (int k = 0; k < kDecPrepCtas; ++k) v[k] = cl.map_shared_rank(s_share, k)[i];
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < kDecPrepCtas; ++k) t += v[k];
    u[i] = t;
  }
  cl.sync();  // every CTA keeps its shared memory until the others have read it
}

}  // namespace qnf4
