// Forward of the QLoRA linear layer at decode sizes (M <= 16 tokens):
//
//   h[m, n] = sum_k x[m, k] What[n, k] + s sum_j B[n, j] u[j, m],   u = A x^T
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (Heng's Blog), opening formula
// h = dequant(W0) x + (alpha / r) B A x, with What the NF4 weight dequantized through
// its two-level constant (贡献二 Double Quantization: c = e4m3(code2) scale2 + mean).
//
// At M <= 16 the layer is bound by the stream of packed weights (about 4.13 bits per
// parameter), and every weight element is used by at most 16 tokens. The kernel gives
// each warp its own weight tiles and tensor-core work, with no hand-off between warps.
// One launch serves 1 to 8 independent layers (the single-layer forward is n = 1):
//
// * Work: the layers' 16-row blocks form one list of units; CTA p takes a contiguous run
//   of units carrying about 1 / P of the packed bytes, and works through it in segments
//   of at most kDecMaxRb blocks of one layer, each over that layer's whole contraction,
//   so no two CTAs share an output. The 12 compute warps split the 64-column blocks of
//   a segment: warp w takes blocks w, w + 12, ... for all the segment's rows, so each
//   token fragment it loads serves every one of those rows.
// * Loads: the CTA streams its segments through a ring of stages in shared memory (as
//   many as fit, 2 to 4), one stage per 12 column blocks (768 columns), each filled by
//   TMA tile copies from a producer warp of its own (warp 12), which refills a stage as
//   soon as the 12 compute warps have released it (an "empty" barrier per stage; no
//   CTA-wide barrier in the loop; the producer issues only after the CTA has set up its
//   barriers, and leaves once everything is issued): the packed rows as one box of a
//   3-D view [row][128-byte group][128 bytes] when K is a multiple of 256 (each row's
//   384 bytes requested in order), else as three 128-byte-wide boxes, and the M token
//   rows as one box of a 3-D view of x, [column block][token row][64 columns]; every
//   box uses the 128-byte swizzle. Warp w works on block w of the stage; token columns
//   past M read row M - 1 (they only feed output columns that are never stored).
// * Rows: within each 16-row block, mma row g reads packed row 2 (g mod 4) + g / 4 (and
//   that + 8), which spreads a quarter warp's 8-byte reads over the swizzled pieces.
//   Twelve compute warps (not 16) keep four warps per SM sub-partition, so each thread
//   can hold 128 registers and keep more table lookups in flight.
// * Math: mma.sync m16n8k16 (bf16 in, fp32 out) with the weight rows as the M side and
//   the tokens as N. Within a block the contraction order is permuted, identically for
//   both operands, so that thread t of a quad holds columns 16t .. 16t + 15: its weight
//   fragment is 8 consecutive packed bytes of each of its two rows, turned into bf16
//   pairs by a 256-entry table (one copy per lane, so the lookups never conflict), and
//   its token fragment is 32 consecutive bytes of each of its token rows. The block's
//   partial sums (unscaled levels) are multiplied by the block constant c in fp32 and
//   added to the accumulator.
// * Reduction: at the end of a segment the 12 warps' accumulators are summed in shared
//   memory in a fixed order; the epilogue adds s B u and writes bf16. The producer keeps
//   streaming the next segment meanwhile.
// * Adapter: u = A x^T comes from k_lora_u, launched just before as the primary of a
//   programmatic dependent launch: the main kernel streams its weights while u is
//   computed, and waits for it (griddepcontrol.wait) only before its epilogue.
#pragma once
#include "common.cuh"

namespace qnf4 {

constexpr int kDecWarps = 12;                  // compute warps
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecBlockThreads = kDecThreads + 32;  // plus the producer warp
constexpr int kDecMaxRb = 5;      // 16-row blocks a CTA holds at most
constexpr int kDecMaxRows = 16 * kDecMaxRb;
constexpr int kDecMaxStages = 4;
constexpr int kDecSbBlocks = kDecWarps;     // column blocks per stage (one per warp)
constexpr int kDecGroups = kDecSbBlocks / 4;  // 128-byte packed groups per stage row
static_assert(kDecSbBlocks % 4 == 0, "a stage holds whole 128-byte packed groups");
constexpr uint32_t kDecRingBytes = 152u * 1024u;
constexpr int kDecLutCopies = 32;
constexpr int kDecRedSlots = 4;
constexpr int kDecRedRow = 84;   // floats per token row of a reduction slot (padded)
constexpr uint32_t kDecLutBytes = 256u * kDecLutCopies * 4u;                 // 32 KB
constexpr uint32_t kDecRedBytes = kDecRedSlots * 16u * kDecRedRow * 4u;      // 21 KB
constexpr uint32_t kDecCsBytes = kDecWarps * kDecMaxRows * 4u;               // 5 KB
constexpr uint32_t kDecBsBytes = kDecMaxRows * 64u * 2u;                     // 10 KB: B rows, r <= 64
constexpr uint32_t kDecUsBytes = 64u * 16u * 4u;                             // 4 KB: u [r][M]
constexpr size_t kDecSmem =
    1024 + kDecRingBytes + kDecLutBytes + kDecCsBytes + kDecBsBytes + kDecRedBytes + kDecUsBytes;
// stage = the token box (kDecSbBlocks blocks x M rows x 128 B), then the packed rows
// (kDecGroups x 16R rows x 128 B); both start on a 1024-byte boundary (the swizzle's)
__host__ __device__ constexpr uint32_t dec_x_bytes(int M) {
  return (128u * kDecSbBlocks * M + 1023u) & ~1023u;
}
__host__ __device__ constexpr uint32_t dec_stage_bytes(int R, int M) {
  return dec_x_bytes(M) + ((2048u * kDecGroups * R + 1023u) & ~1023u);
}
__host__ __device__ constexpr int dec_stages(int R, int M) {
  return static_cast<int>(kDecRingBytes / dec_stage_bytes(R, M)) < kDecMaxStages
             ? static_cast<int>(kDecRingBytes / dec_stage_bytes(R, M))
             : kDecMaxStages;
}
static_assert(dec_stages(kDecMaxRb, 16) >= 2, "the ring must hold two stages of the largest tile");
constexpr int kDecUChunk = 1024;  // contraction columns per k_lora_u partial (128 threads x 8)
constexpr int kDecMaxUParts = 64;  // partials (K <= 65536)

constexpr int kDecMaxGroup = 8;    // layers per launch
constexpr int kDecMaxCta = 256;    // CTAs per launch (one per SM)

// One layer of a launch.
struct DecLayer {
  int64_t N, K;
  int nkb, ks, w3d;          // 64-blocks per row, adapter partials, packed boxes are 3-D
  int64_t unit0;             // first unit (16-row block) of this layer in the launch
  int64_t nb2;               // scale2 entries
  const uint8_t* code2;
  const float* scale2;
  const float* mean;
  const uint16_t* x;         // [M, K] bf16
  const uint16_t* A;         // [r, K] bf16
  const uint16_t* Bm;        // [N, r] bf16
  float* upart;              // [ks][r][M] fp32
  uint16_t* h;               // [M, N] bf16
};

struct DecodeArgs {
  // wmap[l][i]: layer l's packed weight in boxes of 16 (i + 1) rows, as [N][K/256][128]
  // bytes in boxes of rows x 4 x 128 (w3d) or as [N, K/2] bytes in boxes of 128 x rows;
  // xmap[l]: x as [K/64][M][64] in boxes of 16 blocks x M rows x 64 columns
  CUtensorMap wmap[kDecMaxGroup][kDecMaxRb];
  CUtensorMap xmap[kDecMaxGroup];
  DecLayer L[kDecMaxGroup];
  int n, M, r;
  float scale;
  float levels[16];
  int64_t units;                  // 16-row blocks of all layers
  int64_t cta_unit[kDecMaxCta + 1];  // CTA p holds units [cta_unit[p], cta_unit[p + 1])
};

QNF4_DEV uint4 lds_u4d(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
QNF4_DEV uint2 lds_u2d(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
QNF4_DEV uint32_t lds_u32d(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// pair table entry of byte i of w: bf16 levels of its high nibble (bits 0-15, the lower
// column) and low nibble (bits 16-31)
QNF4_DEV uint32_t lut_pair(uint32_t lutb, uint32_t w, int i) {
  return lds_u32d(lutb + (__byte_perm(w, 0u, 0x4440u + i) << 7));
}
QNF4_DEV void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                             uint32_t b0, uint32_t b1, const float (&c)[4]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
        "f"(c[3]));
}

// The adapter projections u_l = A_l x_l^T in partial sums over contraction chunks of
// 1024: CTA (j, c, l) writes layer l's upart[c][j][m] for every token m (fixed-order
// reduction over its four warps). Launched as a programmatic dependent of whatever ran
// before: it first waits for that grid, then lets its own dependent (the main kernel)
// start.
__global__ void __launch_bounds__(128) k_lora_u(const __grid_constant__ DecodeArgs g) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float s_red[4][16];
  const int j = blockIdx.x, c = blockIdx.y, l = blockIdx.z;
  const DecLayer& L = g.L[l];
  const int M = g.M, r = g.r;
  const int64_t K = L.K;
  if (c >= L.ks) return;
  const int64_t k0 = static_cast<int64_t>(c) * kDecUChunk + threadIdx.x * 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool in = k0 < K;  // K is a multiple of 64, so k0 + 7 < K too
  uint4 av = make_uint4(0u, 0u, 0u, 0u);
  uint4 xv[16];
  if (in) av = *reinterpret_cast<const uint4*>(L.A + j * K + k0);
#pragma unroll
  for (int m = 0; m < 16; ++m)
    xv[m] = (in && m < M) ? *reinterpret_cast<const uint4*>(L.x + m * K + k0) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
  float vm[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const uint32_t xw[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
    float v = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v = fmaf(bf16lo(aw[e]), bf16lo(xw[e]), v);
      v = fmaf(bf16hi(aw[e]), bf16hi(xw[e]), v);
    }
    vm[m] = v;
  }
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m < M) {
      float v = vm[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) s_red[warp][m] = v;
    }
  }
  __syncthreads();
  if (threadIdx.x < M) {
    const float v = ((s_red[0][threadIdx.x] + s_red[1][threadIdx.x]) + s_red[2][threadIdx.x]) + s_red[3][threadIdx.x];
    const int64_t o = (static_cast<int64_t>(c) * r + j) * M + threadIdx.x;
    L.upart[o] = v;
  }
}

// barrier of the compute warps only (the producer warp has left)
QNF4_DEV void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kDecThreads) : "memory"); }

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros and reads nothing
QNF4_DEV void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
QNF4_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
QNF4_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Q token groups of 8 (Q = 1: M <= 8; Q = 2: M <= 16).
template <int Q>
__global__ void __launch_bounds__(kDecBlockThreads, 1)
    k_nf4_decode(const __grid_constant__ DecodeArgs g, unsigned long long wait_ns) {
  extern __shared__ uint8_t dsm_raw[];
  __shared__ __align__(8) uint64_t full[kDecMaxStages];
  __shared__ __align__(8) uint64_t empty[kDecMaxStages];
  __shared__ volatile int s_abort;
  __shared__ volatile int s_issued;  // stages the producer issued, -1 while it runs
  uint8_t* base = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
  uint8_t* ring = base;
  uint32_t* lut = reinterpret_cast<uint32_t*>(base + kDecRingBytes);
  float* cs_all = reinterpret_cast<float*>(base + kDecRingBytes + kDecLutBytes);
  uint16_t* bs = reinterpret_cast<uint16_t*>(base + kDecRingBytes + kDecLutBytes + kDecCsBytes);
  float* red = reinterpret_cast<float*>(base + kDecRingBytes + kDecLutBytes + kDecCsBytes + kDecBsBytes);
  float* us = red + kDecRedBytes / 4;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t = lane & 3;
  const int pg = 2 * (g8 & 3) + (g8 >> 2);  // packed row of mma row g8 within 8
  const int M = g.M;
  const uint32_t stb = dec_stage_bytes(kDecMaxRb, M);
  const int nst = dec_stages(kDecMaxRb, M);
  const uint32_t woff = dec_x_bytes(M);
  const bool producer = warp == kDecWarps;
  const int64_t u_begin = g.cta_unit[blockIdx.x], u_end = g.cta_unit[blockIdx.x + 1];
  // the segment starting at unit u: layer l, its first row block rb, R <= kDecMaxRb blocks
  auto seg_of = [&](int64_t u, int& l, int64_t& rb, int& R) {
    l = 0;
    while (l + 1 < g.n && g.L[l + 1].unit0 <= u) ++l;
    rb = u - g.L[l].unit0;
    const int64_t lend = l + 1 < g.n ? g.L[l + 1].unit0 : g.units;
    const int64_t e = u_end < lend ? u_end : lend;
    R = static_cast<int>(e - u < kDecMaxRb ? e - u : kDecMaxRb);
  };
  if (tid == 0) {
    s_abort = 0;
    s_issued = -1;
    for (int i = 0; i < kDecMaxStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kDecWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (producer) {
    // stream the CTA's segments: stage gs (a global count) goes into slot gs mod nst
    // once the compute warps have released that slot's previous use; then leave
    if (lane == 0) {
      int64_t gs = 0;
      bool stop = false;
      for (int64_t u = u_begin; u < u_end && !stop;) {
        int l, R;
        int64_t rb;
        seg_of(u, l, rb, R);
        const DecLayer& L = g.L[l];
        const CUtensorMap* wm = &g.wmap[l][R - 1];
        const int nsb = (L.nkb + kDecSbBlocks - 1) / kDecSbBlocks;
        const int32_t row0 = static_cast<int32_t>(rb * 16);
        for (int j = 0; j < nsb; ++j) {
          if (gs >= nst) {
            const long long t0 = wait_clock();
            while (!mbar_try_wait(&empty[gs % nst], static_cast<uint32_t>((gs / nst - 1) & 1))) {
              if (s_abort) {
                stop = true;
                break;
              }
              if (wait_clock() - t0 > ns_cycles(wait_ns)) {
                set_err(63);
                s_abort = 1;
                stop = true;
                break;
              }
            }
            if (stop) break;
            fence_proxy_async();
          }
          if (s_abort) {
            stop = true;
            break;
          }
          uint8_t* st = ring + (gs % nst) * stb;
          uint64_t* bar = &full[gs % nst];
          const int kb0 = j * kDecSbBlocks;
          mbar_expect_tx(bar, 128u * kDecSbBlocks * M + kDecGroups * 16u * R * 128u);
          tma_load_3d(st, &g.xmap[l], bar, 0, 0, kb0);
          if (L.w3d) {
            tma_load_3d(st + woff, wm, bar, 0, kb0 / 4, row0);
          } else {
            for (int b = 0; b < kDecGroups; ++b)
              tma_load_2d(st + woff + b * (16u * R * 128u), wm, bar, kb0 * 32 + b * 128, row0);
          }
          ++gs;
        }
        u += R;
      }
      s_issued = static_cast<int>(gs);
    }
    return;
  }

  // pair table: entry b, copy j at word b * 32 + j
  for (int i = tid; i < 256 * kDecLutCopies; i += kDecThreads) {
    const int b = i / kDecLutCopies;
    lut[i] = pack_bf16x2(g.levels[b >> 4], g.levels[b & 15]);
  }
  compute_sync();

  const uint32_t lutb = smem_u32(lut) + lane * 4u;
  float* cs = cs_all + warp * kDecMaxRows;
  constexpr int kCpl = (kDecMaxRows + 31) / 32;  // rows per lane for the block constants
  bool ok = true, waited = false;
  int ul = -1;  // layer whose u is in us
  int64_t gs = 0;
  for (int64_t u = u_begin; u < u_end;) {
    int l, R;
    int64_t rb;
    seg_of(u, l, rb, R);
    u += R;
    const DecLayer& L = g.L[l];
    const int64_t row0 = rb * 16, N = L.N;
    const int nkb = L.nkb;
    const int nsb = (nkb + kDecSbBlocks - 1) / kDecSbBlocks;
    const float mu = __ldg(L.mean);
    const bool w3d = L.w3d != 0;
    const uint8_t* __restrict__ code2 = L.code2;
    const float* __restrict__ scale2 = L.scale2;
    // this segment's rows of B (bf16 [16R, r]) for its epilogue: asynchronous 16-byte
    // copies when the rows are 16-byte aligned (r a multiple of 8), else plain loads
    const int r = g.r;
    if ((r & 7) == 0) {
      const int np = 16 * R * r / 8;
      for (int i = tid; i < np; i += kDecThreads) {
        const int64_t n = row0 + (i * 8) / r;
        const bool in = n < N;
        cp_async16(smem_u32(bs + i * 8), in ? L.Bm + row0 * r + i * 8 : L.Bm, in ? 16u : 0u);
      }
      cp_async_commit();
    } else {
      for (int i = tid; i < 16 * R * r; i += kDecThreads) {
        const int64_t n = row0 + i / r;
        bs[i] = n < N ? L.Bm[n * r + i % r] : static_cast<uint16_t>(0);
      }
    }
    // block constants (code2 byte, scale2) of rows lane + 32 c for this warp's block of
    // stage j, loaded one stage ahead of their use
    // the block index of this lane's rows at block 0 (or -1 past the rows)
    int64_t cblk[kCpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) {
      const int rr = lane + 32 * c;
      cblk[c] = (rr < 16 * R && row0 + rr < N) ? (row0 + rr) * nkb + warp : -1;
    }
    auto cload = [&](int j, uint32_t (&q)[kCpl], float (&sc)[kCpl]) {
      const bool live = j < nsb && j * kDecSbBlocks + warp < nkb;
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        q[c] = 0u;
        sc[c] = 0.f;
        const int64_t blk = cblk[c] + j * kDecSbBlocks;
        if (live && cblk[c] >= 0 && in_bounds((blk >> 8) < L.nb2, 71)) {
          q[c] = code2[blk];
          sc[c] = scale2[blk >> 8];
        }
      }
    };
    uint32_t pq[kCpl];
    float psc[kCpl];
    cload(0, pq, psc);
    float acc[kDecMaxRb][Q][4];
#pragma unroll
    for (int b = 0; b < kDecMaxRb; ++b)
#pragma unroll
      for (int q = 0; q < Q; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[b][q][e] = 0.f;
    const uint32_t gg = warp >> 2;
    const uint32_t u0 = 2u * (warp & 3) + (t >> 1);
    // this warp's 32 packed bytes of row rr: 128-byte group warp / 4, pieces 2 (warp mod
    // 4) and + 1, swizzled by the 128-byte line: line = rr * 4 + group (3-D boxes) or
    // group * 16R + rr (four 2-D boxes). Rows pg + 16 b (+ 8) share the line's swizzle
    // key, so row block b sits at a fixed stride from row block 0.
    const uint32_t la0 = w3d ? static_cast<uint32_t>(pg) * kDecGroups + gg : gg * 16u * R + static_cast<uint32_t>(pg);
    const uint32_t woffa = woff + la0 * 128u + (((u0 ^ (la0 & 7u)) << 4) | ((t & 1) << 3));
    const uint32_t bstride = w3d ? 16u * kDecGroups * 128u : 16u * 128u;  // bytes per row block
    const uint32_t hstride = bstride / 2;                          // rows + 8
    // token fragment offsets (rows g8, g8 + 8 of this warp's block, the last row past M)
    uint32_t xoffa[Q], xoffb[Q];
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const int tr = g8 + 8 * q < M ? g8 + 8 * q : M - 1;
      const uint32_t rho = static_cast<uint32_t>(warp * M + tr);
      xoffa[q] = rho * 128u + ((static_cast<uint32_t>(2 * t) ^ (rho & 7u)) << 4);
      xoffb[q] = rho * 128u + ((static_cast<uint32_t>(2 * t + 1) ^ (rho & 7u)) << 4);
    }
    for (int j = 0; j < nsb; ++j, ++gs) {
      if (ok) ok = warp_wait(&full[gs % nst], static_cast<uint32_t>((gs / nst) & 1), wait_ns, &s_abort, 61);
      if (!ok) continue;  // after a give-up no stage is released: the producer stops
      const int kb = j * kDecSbBlocks + warp;
      if (kb >= nkb) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[gs % nst]);
        continue;
      }
      const uint32_t sb = smem_u32(ring + (gs % nst) * stb);
      // c of the segment's rows for block kb, exchanged through the warp's scratch:
      // packed row rr at word (rr mod 8) * 2 kDecMaxRb + rr / 8, so thread (g8, t) reads
      // its rows pg + 8 i at pg * 2 kDecMaxRb + i
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        const int rr = lane + 32 * c;
        if (rr < kDecMaxRows)
          cs[(rr & 7) * (2 * kDecMaxRb) + (rr >> 3)] =
              fmaf(e4m3_to_f32(static_cast<uint8_t>(pq[c])), psc[c], mu);
      }
      cload(j + 1, pq, psc);  // the next stage's constants land while the tensor cores work
      __syncwarp();
      float ch[2 * kDecMaxRb];
#pragma unroll
      for (int i = 0; i < kDecMaxRb; ++i) {
        const float2 v = *reinterpret_cast<const float2*>(cs + pg * (2 * kDecMaxRb) + 2 * i);
        ch[2 * i] = v.x;
        ch[2 * i + 1] = v.y;
      }
      // token fragments: row g8 (+ 8), columns 16 t .. 16 t + 15 of this warp's block
      // (row rho = warp M + row of the box, pieces 2t, 2t+1 swizzled by rho mod 8)
      uint4 xa[Q], xb[Q];
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        xa[q] = lds_u4d(sb + xoffa[q]);
        xb[q] = lds_u4d(sb + xoffb[q]);
      }
      const uint32_t wbase = sb + woffa;
      const float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int b = 0; b < kDecMaxRb; ++b) {
        if (b < R) {
          const uint2 wa = lds_u2d(wbase + b * bstride);
          const uint2 wb = lds_u2d(wbase + b * bstride + hstride);
          float d[Q][4];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t wlo = k4 < 2 ? wa.x : wa.y, whi = k4 < 2 ? wb.x : wb.y;
            const int i0 = (2 * k4) & 3;
            const uint32_t a0 = lut_pair(lutb, wlo, i0), a2 = lut_pair(lutb, wlo, i0 + 1);
            const uint32_t a1 = lut_pair(lutb, whi, i0), a3 = lut_pair(lutb, whi, i0 + 1);
#pragma unroll
            for (int q = 0; q < Q; ++q) {
              const uint4& xv = k4 < 2 ? xa[q] : xb[q];
              const uint32_t b0 = (k4 & 1) ? xv.z : xv.x, b1 = (k4 & 1) ? xv.w : xv.y;
              if (k4 == 0)
                mma_bf16_16816(d[q], a0, a1, a2, a3, b0, b1, z);
              else
                mma_bf16_16816(d[q], a0, a1, a2, a3, b0, b1, d[q]);
            }
          }
#pragma unroll
          for (int q = 0; q < Q; ++q) {
            acc[b][q][0] = fmaf(ch[2 * b], d[q][0], acc[b][q][0]);
            acc[b][q][1] = fmaf(ch[2 * b], d[q][1], acc[b][q][1]);
            acc[b][q][2] = fmaf(ch[2 * b + 1], d[q][2], acc[b][q][2]);
            acc[b][q][3] = fmaf(ch[2 * b + 1], d[q][3], acc[b][q][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[gs % nst]);  // this warp is done with the stage
    }
    if (!ok) break;

    // ---- segment end: u of this layer (once the adapter kernel has finished), the
    // fixed-order sum of the compute warps' partials (warp w adds into slot w % 4, warps 0-3
    // first, then 4-7 and 8-11; slots [token][row], rows padded to kDecRedRow) ----
    if (!waited) {
      griddep_wait();
      waited = true;
    }
    const int nu = r * M;
    const bool newu = l != ul;
    float up[kDecMaxUParts / 4];
    if (newu) {
#pragma unroll
      for (int c = 0; c < kDecMaxUParts / 4; ++c)
        up[c] = (tid < nu && c < L.ks) ? __ldcg(L.upart + static_cast<int64_t>(c) * nu + tid) : 0.f;
    }
    float* slot = red + (warp % kDecRedSlots) * (16 * kDecRedRow);
#pragma unroll
    for (int round = 0; round < kDecWarps / kDecRedSlots; ++round) {
      if (warp / kDecRedSlots == round) {
#pragma unroll
        for (int b = 0; b < kDecMaxRb; ++b) {
          if (b < R) {
#pragma unroll
            for (int q = 0; q < Q; ++q) {
              const int rw = b * 16 + pg, tk = 8 * q + 2 * t;  // the packed row of mma row g8
              float* p = slot + tk * kDecRedRow + rw;
              if (round == 0) {
                p[0] = acc[b][q][0];
                p[kDecRedRow] = acc[b][q][1];
                p[8] = acc[b][q][2];
                p[kDecRedRow + 8] = acc[b][q][3];
              } else {
                p[0] += acc[b][q][0];
                p[kDecRedRow] += acc[b][q][1];
                p[8] += acc[b][q][2];
                p[kDecRedRow + 8] += acc[b][q][3];
              }
            }
          }
        }
      }
      compute_sync();
    }
    if (newu) {
      for (int i = tid; i < nu; i += kDecThreads) {
        float v = 0.f;
        if (i == tid) {
#pragma unroll
          for (int c = 0; c < kDecMaxUParts / 4; ++c) v += up[c];
        } else {
          for (int c = 0; c < kDecMaxUParts / 4 && c < L.ks; ++c)
            v += __ldcg(L.upart + static_cast<int64_t>(c) * nu + i);
        }
        for (int c = kDecMaxUParts / 4; c < L.ks; ++c) v += __ldcg(L.upart + static_cast<int64_t>(c) * nu + i);
        us[i] = v;
      }
      ul = l;
    }
    cp_async_wait_all();  // the B rows
    compute_sync();
    // outputs o = m * 16 R + row: h[m, row0 + row] = sum of the slots + s B u
    const int nrows = 16 * R;
    const int nout = nrows * M;
    for (int o = tid; o < nout; o += kDecThreads) {
      const int rl = o % nrows, m = o / nrows;
      const int64_t n = row0 + rl;
      if (n >= N) continue;
      float v = 0.f;
#pragma unroll
      for (int sl = 0; sl < kDecRedSlots; ++sl) v += red[sl * (16 * kDecRedRow) + m * kDecRedRow + rl];
      const uint16_t* brow = bs + rl * r;
      float lr = 0.f;
      if ((r & 7) == 0) {
        for (int j = 0; j < r; j += 8) {
          const uint4 bv = *reinterpret_cast<const uint4*>(brow + j);
          const float* uj = us + j * M + m;
          lr = fmaf(bf16lo(bv.x), uj[0], lr);
          lr = fmaf(bf16hi(bv.x), uj[M], lr);
          lr = fmaf(bf16lo(bv.y), uj[2 * M], lr);
          lr = fmaf(bf16hi(bv.y), uj[3 * M], lr);
          lr = fmaf(bf16lo(bv.z), uj[4 * M], lr);
          lr = fmaf(bf16hi(bv.z), uj[5 * M], lr);
          lr = fmaf(bf16lo(bv.w), uj[6 * M], lr);
          lr = fmaf(bf16hi(bv.w), uj[7 * M], lr);
        }
      } else {
        for (int j = 0; j < r; ++j) lr = fmaf(bf16lo(brow[j]), us[j * M + m], lr);
      }
      const float out = fmaf(g.scale, lr, v);
      if (in_bounds(m < M, 74))
        L.h[static_cast<int64_t>(m) * N + n] = static_cast<uint16_t>(pack_bf16x2(out, 0.f) & 0xFFFFu);
    }
    compute_sync();  // red, us and bs are reused by the next segment
  }
  // Drain: after a give-up, the stages issued but not waited for must land before the
  // CTA exits (one deadline). At most nst stages can be in flight, each in its own slot.
  compute_sync();
  if (tid == 0 && s_abort) {
    const long long t0 = wait_clock();
    while (s_issued < 0 && wait_clock() - t0 <= ns_cycles(drain_ns(wait_ns))) {
    }
    const int issued = s_issued < 0 ? 0 : s_issued;
    for (int jj = issued - nst > 0 ? issued - nst : 0; jj < issued; ++jj) {
      while (!mbar_try_wait_long(&full[jj % nst], static_cast<uint32_t>((jj / nst) & 1))) {
        if (wait_clock() - t0 > ns_cycles(drain_ns(wait_ns))) {
          set_err(62);
          break;
        }
      }
    }
  }
  cp_async_wait_all();
}

}  // namespace qnf4
