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
//   of at most 5 blocks of one layer (4 with two token groups, whose accumulators and
//   token fragments are twice as many), each over that layer's whole contraction, so no
//   two CTAs share an output. The 12 compute warps split the 64-column blocks of a
//   segment: warp w takes blocks w, w + 12, ... for all the segment's rows, so each token
//   fragment it loads serves every one of those rows. The row-block count of a segment is
//   a compile-time constant of its loop (one instance per count), so the row blocks'
//   table lookups interleave without branches.
// * Loads: the CTA streams its segments through a ring of stages in shared memory (as
//   many as fit, 2 to 4), one stage per 12 column blocks (768 columns). Two producer
//   warps walk the same stages and refill a slot as soon as the 12 compute warps have
//   released it (an "empty" barrier per stage; no CTA-wide barrier in the loop). Warp 12
//   issues the TMA tile copies: the packed rows as one box of a 3-D view [row][128-byte
//   group][128 bytes] when K is a multiple of 256 (each row's 384 bytes requested in
//   order), else as three 128-byte-wide boxes, and the M token rows as one box of a 3-D
//   view of x, [column block][token row][64 columns]; every box uses the 128-byte
//   swizzle. Warp 13 copies the stage's block constants (per row, the code2 bytes of its
//   12 blocks and the two scale2 words they can use) with 4-byte asynchronous copies and
//   arrives on the stage's barrier when they land, so the tile copies never queue behind
//   those small ones. Warp w works on block w of the stage; token columns past M read
//   row M - 1 (they only feed output columns that are never stored).
// * Rows: within each 16-row block, mma row g reads packed row 2 (g mod 4) + g / 4 (and
//   that + 8), which spreads a quarter warp's 8-byte reads over the swizzled pieces.
//   Twelve compute warps (not 16) keep at most four warps per SM sub-partition, so each
//   thread can hold 128 registers and keep more table lookups in flight.
// * Math: mma.sync m16n8k16 (bf16 in, fp32 out) with the weight rows as the M side and
//   the tokens as N. Within a block the contraction order is permuted, identically for
//   both operands, so that thread t of a quad holds columns 16t .. 16t + 15: its weight
//   fragment is 8 consecutive packed bytes of each of its two rows, turned into bf16
//   pairs by a 256-entry table (one copy per lane, so the lookups never conflict), and
//   its token fragment is 32 consecutive bytes of each of its token rows. The block's
//   partial sums (unscaled levels) are multiplied by the block constant c (computed per
//   stage from the staged code2 and scale2) in fp32 and added to the accumulator.
// * Reduction: at the end of a segment the 12 warps' accumulators are summed in shared
//   memory in a fixed order and written as bf16. Warp 0 first adds the adapter term
//   s B u to its accumulators with the same tensor-core instruction (B rows and bf16 s u
//   in shared memory, the rank padded to a multiple of 16 with zeros). The producers
//   keep streaming the next segment meanwhile.
// * Adapter: u = A x^T comes from k_lora_u, launched just before as the primary of a
//   programmatic dependent launch: the main kernel streams its weights while u is
//   computed, and waits for it (griddepcontrol.wait) only before its first epilogue.
#pragma once
#include "common.cuh"

namespace qnf4 {

constexpr int kDecWarps = 12;                  // compute warps
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecBlockThreads = kDecThreads + 64;  // plus the two producer warps
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
constexpr uint32_t kDecCsBytes = kDecWarps * kDecMaxRows * 4u;               // 4 KB
constexpr uint32_t kDecBsBytes = kDecMaxRows * 64u * 2u;                     // 10 KB: B rows, r <= 64
constexpr uint32_t kDecUsBytes = 16u * 64u * 2u;                             // 2 KB: bf16 s u [token][r]
constexpr size_t kDecSmem =
    1024 + kDecRingBytes + kDecLutBytes + kDecCsBytes + kDecBsBytes + kDecRedBytes + kDecUsBytes;
// Block constants of a stage, copied by the producer warp: for each of the 16R rows the
// 16 code2 bytes from its first block's byte rounded down to 4 (the stage's 12 blocks lie
// inside), then the two scale2 words its 12 blocks can fall into.
constexpr uint32_t kDecCodeRow = 16u;
constexpr uint32_t kDecCstScale = kDecMaxRows * kDecCodeRow;                 // 1280
constexpr uint32_t kDecCstBytes = 2048u;
static_assert(kDecCstScale + kDecMaxRows * 8u <= kDecCstBytes, "constants area");
// stage = the token box (kDecSbBlocks blocks x M rows x 128 B), the packed rows
// (kDecGroups x 16R rows x 128 B), then the block constants; the boxes start on a
// 1024-byte boundary (the swizzle's)
__host__ __device__ constexpr uint32_t dec_x_bytes(int M) {
  return (128u * kDecSbBlocks * M + 1023u) & ~1023u;
}
__host__ __device__ constexpr uint32_t dec_w_bytes(int R) {
  return (2048u * kDecGroups * R + 1023u) & ~1023u;
}
__host__ __device__ constexpr uint32_t dec_stage_bytes(int R, int M) {
  return dec_x_bytes(M) + dec_w_bytes(R) + kDecCstBytes;
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
  // bytes in boxes of rows x kDecGroups x 128 (w3d) or as [N, K/2] bytes in boxes of
  // 128 x rows; xmap[l]: x as [K/64][M][64] in boxes of kDecSbBlocks blocks x M rows x 64
  // columns
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
// 4-byte asynchronous copy global -> shared of src_bytes (0..4) bytes, the rest zeros
QNF4_DEV void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
QNF4_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
QNF4_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// one arrival on the barrier once this thread's earlier cp.async copies have landed
// (counted among the barrier's expected arrivals)
QNF4_DEV void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
QNF4_DEV uint32_t lds_u8d(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
QNF4_DEV float lds_f32d(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

template <int V>
struct DecRows {
  static constexpr int value = V;
};

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
  uint16_t* us = reinterpret_cast<uint16_t*>(red + kDecRedBytes / 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t = lane & 3;
  const int pg = 2 * (g8 & 3) + (g8 >> 2);  // packed row of mma row g8 within 8
  const int M = g.M;
  // row blocks per segment: two token groups keep fewer (their accumulators and token
  // fragments are twice as many), which also leaves room for a third stage
  constexpr int kRb = Q == 2 ? 4 : kDecMaxRb;
  const uint32_t stb = dec_stage_bytes(kRb, M);
  const int nst = dec_stages(kRb, M);
  const uint32_t woff = dec_x_bytes(M);
  const uint32_t coff = woff + dec_w_bytes(kRb);  // block constants of a stage
  const bool producer = warp >= kDecWarps;
  const int64_t u_begin = g.cta_unit[blockIdx.x], u_end = g.cta_unit[blockIdx.x + 1];
  // the segment starting at unit u: layer l, its first row block rb, R <= kRb blocks
  auto seg_of = [&](int64_t u, int& l, int64_t& rb, int& R) {
    l = 0;
    while (l + 1 < g.n && g.L[l + 1].unit0 <= u) ++l;
    rb = u - g.L[l].unit0;
    const int64_t lend = l + 1 < g.n ? g.L[l + 1].unit0 : g.units;
    const int64_t e = u_end < lend ? u_end : lend;
    R = static_cast<int>(e - u < kRb ? e - u : kRb);
  };
  if (tid == 0) {
    s_abort = 0;
    s_issued = -1;
    for (int i = 0; i < kDecMaxStages; ++i) {
      mbar_init(&full[i], 1 + 32);  // the tile warp's transaction + the constant warp's 32 lanes
      mbar_init(&empty[i], kDecWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (producer) {
    // stream the CTA's segments: stage gs (a global count) goes into slot gs mod nst
    // once the compute warps have released that slot's previous use. Both producer warps
    // walk the same stages: lane 0 of warp 12 issues the tile copies, the lanes of warp
    // 13 copy the block constants and arrive on the stage's barrier when they have
    // landed (so the tile copies never queue behind the many small ones).
    const bool tma_warp = warp == kDecWarps;
    int64_t gs = 0;
    bool stop = false;
    for (int64_t u = u_begin; u < u_end && !stop;) {
      int l, R;
      int64_t rb;
      seg_of(u, l, rb, R);
      const DecLayer& L = g.L[l];
      const CUtensorMap* wm = &g.wmap[l][R - 1];
      const int nkb = L.nkb;
      const int nsb = (nkb + kDecSbBlocks - 1) / kDecSbBlocks;
      const int32_t row0 = static_cast<int32_t>(rb * 16);
      const int64_t c2len = L.N * nkb;  // code2 bytes
      int64_t crow[(kDecMaxRows + 31) / 32];  // block index of this lane's rows at column 0
#pragma unroll
      for (int c = 0; c < (kDecMaxRows + 31) / 32; ++c) crow[c] = (row0 + lane + 32 * c) * static_cast<int64_t>(nkb);
      for (int j = 0; j < nsb; ++j) {
        const int slot = static_cast<int>(gs % nst);
        if (gs >= nst) {
          if (!warp_wait(&empty[slot], static_cast<uint32_t>((gs / nst - 1) & 1), wait_ns, &s_abort, 63)) {
            stop = true;
            break;
          }
          fence_proxy_async();
        }
        if (__shfl_sync(0xffffffffu, s_abort, 0)) {
          stop = true;
          break;
        }
        uint8_t* st = ring + slot * stb;
        uint64_t* bar = &full[slot];
        const int kb0 = j * kDecSbBlocks;
        if (tma_warp && lane == 0) {
          mbar_expect_tx(bar, 128u * kDecSbBlocks * M + kDecGroups * 16u * R * 128u);
          tma_load_3d(st, &g.xmap[l], bar, 0, 0, kb0);
          if (L.w3d) {
            tma_load_3d(st + woff, wm, bar, 0, kb0 / 4, row0);
          } else {
            for (int b = 0; b < kDecGroups; ++b)
              tma_load_2d(st + woff + b * (16u * R * 128u), wm, bar, kb0 * 32 + b * 128, row0);
          }
        }
        if (!tma_warp) {
          // block constants: lane handles rows lane + 32 c: 4 code2 words from the row's
          // first block rounded down to 4 bytes (the last word of code2 may be partial), then
          // scale2 words s0 and s0 + 1
          const uint32_t cdst = smem_u32(st + coff);
#pragma unroll
          for (int c = 0; c < (kDecMaxRows + 31) / 32; ++c) {
            const int rr = lane + 32 * c;
            if (rr < 16 * R) {
              const bool live = row0 + rr < L.N;
              const int64_t a = crow[c] + kb0;
              const int64_t w0 = a & ~static_cast<int64_t>(3);
              const int64_t left = live ? c2len - w0 : 0;
              const uint32_t d = cdst + rr * kDecCodeRow;
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const int64_t lv = left - 4 * v;
                const uint32_t nb = lv >= 4 ? 4u : (lv > 0 ? static_cast<uint32_t>(lv) : 0u);
                cp_async4(d + 4 * v, nb ? L.code2 + w0 + 4 * v : L.code2, nb);
              }
              const int64_t s0 = a >> 8;
              const uint32_t ds = cdst + kDecCstScale + rr * 8;
              cp_async4(ds, live ? L.scale2 + s0 : L.scale2, live ? 4u : 0u);
              const bool ok1 = live && s0 + 1 < L.nb2;
              cp_async4(ds + 4, ok1 ? L.scale2 + s0 + 1 : L.scale2, ok1 ? 4u : 0u);
              in_bounds(!live || (w0 >= 0 && s0 < L.nb2), 75);
            }
          }
          cp_async_mbar_arrive(bar);
        }
        ++gs;
      }
      u += R;
    }
    if (tma_warp && lane == 0) s_issued = static_cast<int>(gs);
    cp_async_wait_all();
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
  const int r = g.r;
  const int r16 = (r + 15) & ~15;  // the adapter's contraction, padded with zeros
  bool ok = true, waited = false;
  int ul = -1;  // layer whose s u is in us
  int64_t gs = 0;
  // one segment of R row blocks (R a compile-time constant, so the row-block loops
  // unroll without branches and their table lookups interleave)
  auto segment = [&](auto Rc, int l, int64_t rb) {
    constexpr int R = decltype(Rc)::value;
    const DecLayer& L = g.L[l];
    const int64_t row0 = rb * 16, N = L.N;
    const int nkb = L.nkb;
    const int nsb = (nkb + kDecSbBlocks - 1) / kDecSbBlocks;
    const float mu = __ldg(L.mean);
    const bool w3d = L.w3d != 0;
    // this segment's rows of B as bf16 [16R][r16] (zero past r and past N) for the
    // adapter product: 16-byte asynchronous copies when rows are 16-byte aligned
    if ((r & 7) == 0) {
      const int pr = r16 / 8;
      for (int i = tid; i < 16 * R * pr; i += kDecThreads) {
        const int rl = i / pr, p = i - pr * (i / pr);
        const int64_t n = row0 + rl;
        const bool in = n < N && 8 * p < r;
        cp_async16(smem_u32(bs + rl * r16 + 8 * p), in ? L.Bm + n * r + 8 * p : L.Bm, in ? 16u : 0u);
      }
      cp_async_commit();
    } else {
      for (int i = tid; i < 16 * R * r16; i += kDecThreads) {
        const int rl = i / r16, jj = i - r16 * (i / r16);
        const int64_t n = row0 + rl;
        bs[i] = (n < N && jj < r) ? L.Bm[n * r + jj] : static_cast<uint16_t>(0);
      }
    }
    // low 8 bits of the block index of this lane's rows (lane + 32 c) at column 0: they
    // give, per stage, the row's byte in the staged code2 window and its scale2 word
    uint32_t alo[kCpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c)
      alo[c] = static_cast<uint32_t>(((row0 + lane + 32 * c) * nkb) & 255);
    float acc[R][Q][4];
#pragma unroll
    for (int b = 0; b < R; ++b)
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
      // c of the segment's rows for block kb from the staged constants, exchanged through
      // the warp's scratch: packed row rr at word (rr mod 8) * 2 kDecMaxRb + rr / 8, so
      // thread (g8, t) reads its rows pg + 8 i at pg * 2 kDecMaxRb + i
      const uint32_t cst = sb + coff;
#pragma unroll
      for (int c = 0; c < kCpl; ++c) {
        const int rr = lane + 32 * c;
        if (rr < 16 * R) {
          const uint32_t a = (alo[c] + static_cast<uint32_t>(j * kDecSbBlocks)) & 255u;
          const uint32_t code = lds_u8d(cst + rr * kDecCodeRow + (a & 3u) + warp);
          const float s2 = lds_f32d(cst + kDecCstScale + rr * 8 + (((a + warp) >> 8) << 2));
          cs[(rr & 7) * (2 * kDecMaxRb) + (rr >> 3)] = fmaf(e4m3_to_f32(static_cast<uint8_t>(code)), s2, mu);
        }
      }
      __syncwarp();
      float ch[2 * R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
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
      for (int b = 0; b < R; ++b) {
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[gs % nst]);  // this warp is done with the stage
    }
    if (!ok) return;

    // ---- segment end: s u of this layer as bf16 [token][r16] (once the adapter kernel
    // has finished; partials summed in a fixed order), then the fixed-order sum of the
    // compute warps' partials (warp w adds into slot w % 4, warps 0-3 first, then 4-7
    // and 8-11; slots [token][row], rows padded to kDecRedRow). Warp 0 first adds the
    // adapter term s B u to its accumulators with the tensor cores. ----
    if (!waited) {
      griddep_wait();
      waited = true;
    }
    if (l != ul) {
      const int nu = r * M;
      for (int i = tid; i < 16 * r16; i += kDecThreads) {
        const int m = i / r16, jj = i - r16 * (i / r16);
        float v = 0.f;
        if (m < M && jj < r) {
          const float* p = L.upart + jj * M + m;
          constexpr int kPre = 8;  // partials loaded together
          for (int c0 = 0; c0 < L.ks; c0 += kPre) {
            float up[kPre];
#pragma unroll
            for (int c = 0; c < kPre; ++c)
              up[c] = c0 + c < L.ks ? __ldcg(p + static_cast<int64_t>(c0 + c) * nu) : 0.f;
#pragma unroll
            for (int c = 0; c < kPre; ++c)
              if (c0 + c < L.ks) v += up[c];
          }
        }
        us[i] = static_cast<uint16_t>(pack_bf16x2(g.scale * v, 0.f) & 0xFFFFu);
      }
      ul = l;
    }
    cp_async_wait_all();  // the B rows
    compute_sync();
    if (warp == 0) {
      const uint32_t bsa = smem_u32(bs), usa = smem_u32(us);
      for (int kc = 0; kc < r16; kc += 16) {
        uint32_t bu[Q][2];
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          const uint32_t o = ((8 * q + g8) * r16 + kc + 2 * t) * 2;
          bu[q][0] = lds_u32d(usa + o);
          bu[q][1] = lds_u32d(usa + o + 16);
        }
#pragma unroll
        for (int b = 0; b < R; ++b) {
          const uint32_t o0 = ((b * 16 + pg) * r16 + kc + 2 * t) * 2;
          const uint32_t o1 = o0 + 8 * r16 * 2;
          const uint32_t a0 = lds_u32d(bsa + o0), a2 = lds_u32d(bsa + o0 + 16);
          const uint32_t a1 = lds_u32d(bsa + o1), a3 = lds_u32d(bsa + o1 + 16);
#pragma unroll
          for (int q = 0; q < Q; ++q) mma_bf16_16816(acc[b][q], a0, a1, a2, a3, bu[q][0], bu[q][1], acc[b][q]);
        }
      }
    }
    float* slot = red + (warp % kDecRedSlots) * (16 * kDecRedRow);
#pragma unroll
    for (int round = 0; round < kDecWarps / kDecRedSlots; ++round) {
      if (warp / kDecRedSlots == round) {
#pragma unroll
        for (int b = 0; b < R; ++b) {
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
      compute_sync();
    }
    // outputs o = m * 16 R + row: h[m, row0 + row] = the slots' sum
    constexpr int nrows = 16 * R;
    for (int o = tid; o < nrows * M; o += kDecThreads) {
      const int rl = o % nrows, m = o / nrows;
      const int64_t n = row0 + rl;
      if (n >= N) continue;
      const float* p = red + m * kDecRedRow + rl;
      const float v = ((p[0] + p[16 * kDecRedRow]) + p[2 * 16 * kDecRedRow]) + p[3 * 16 * kDecRedRow];
      if (in_bounds(m < M, 74))
        L.h[static_cast<int64_t>(m) * N + n] = static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);
    }
    compute_sync();  // red, us and bs are reused by the next segment
  };
  static_assert(kDecMaxRb == 5 && kDecRedSlots == 4, "segment dispatch and slot sum");
  for (int64_t u = u_begin; u < u_end && ok;) {
    int l, R;
    int64_t rb;
    seg_of(u, l, rb, R);
    u += R;
    switch (R) {
      case 1: segment(DecRows<1>{}, l, rb); break;
      case 2: segment(DecRows<2>{}, l, rb); break;
      case 3: segment(DecRows<3>{}, l, rb); break;
      case 4: segment(DecRows<4>{}, l, rb); break;
      default: segment(DecRows<kRb>{}, l, rb); break;
    }
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
