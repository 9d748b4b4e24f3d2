// Grouped, persistent tcgen05 GEMM for sm_100a.
//
// D = A * B^T over many problems at once, one CTA per SM walking a linear tile
// space with a static stride.  Two ways of describing the problems:
//
//   class mode  (GemmParams)  problems are grouped into "classes" of identical
//               (M, N, K); a class's operands are 3-D tensors [count][rows][cols]
//               reached through one TMA descriptor each (kernel parameters), so a
//               batch of hundreds of same-shape matrices costs two descriptors.
//               bf16 epilogues for Newton-Schulz (EPI_GRAM / EPI_POLY / EPI_AXPY_T)
//               and an fp32 store (EPI_STORE_F32).
//   table mode  (GemmTableParams) one entry per problem in a device array, each
//               with its own descriptors in global memory (operands are separate
//               buffers), SPLIT3 operands and an fp32 epilogue
//                   out = alpha * acc + beta * aux          (aux optional, may alias out)
//               that can also emit the three bf16 planes of `out` for a following
//               fp32-faithful product.  A problem can be gated by a device flag
//               (skipped when the flag is 0) for data-dependent work.
//
// Warp roles (320 threads):
//   warp 0      TMA producer (one elected lane): fills a STAGES-deep ring of
//               A/B tiles in shared memory, 128-byte swizzled.
//   warp 1      TMEM owner + MMA issuer (one elected lane): tcgen05.mma into one
//               of two TMEM accumulators (BN fp32 columns each); commits free the
//               smem slots and hand finished accumulators to the epilogue.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = tile rows), fused arithmetic, stores; two
//               warps share each lane quarter, half the tile's columns each.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile i+1.
//
// Operand kinds:
//   BF16    kind::f16, bf16 operands, fp32 accumulate, BK = 64 (128 B rows).
//   SPLIT3  fp32-faithful product on the bf16 tensor cores: each fp32 operand is
//           held as three bf16 planes x = x0 + x1 + x2 (24 significant bits).  The
//           main product x0 y0 accumulates in one fp32 TMEM accumulator and the
//           five cross products whose size reaches the fp32 unit roundoff
//           (x1y1, x0y2, x2y0, x0y1, x1y0) in a second one, so the large running
//           sum is rounded once per k-step only.  The tensor core's accumulation
//           truncates, so its error grows with every add: TMEM accumulates 128 of
//           K at a time (256 for bf16 x bf16) and the epilogue warps fold those
//           partial sums (main + correction) into fp32 registers with
//           round-to-nearest.  Same MMA count per K as a three-pass tf32 scheme,
//           with fp32-level accuracy.
// Operand majors: K-major (rows of the operand run along K) or MN-major
// (rows run along M/N, i.e. the row-major matrix is K x MN).
#pragma once

#include "common.cuh"

namespace mao {

constexpr int kMaxClasses = 8;

enum OperandKind : int { OP_BF16 = 0, OP_SPLIT3 = 1 };

enum EpiKind : int {
  EPI_STORE_F32 = 0,  // out0 (f32) = alpha * acc
  EPI_GRAM = 1,       // out0 (bf16) = acc * s_b^2                    (A = X X^T)
  EPI_POLY = 2,       // out0 (bf16) = beta * aux + gamma * acc       (B = b A + c A A)
  EPI_AXPY_T = 3,     // v = s_b * (alpha * aux + acc); out0 (bf16) = v, out1 = v^T if given  (X = a X + B X)
  EPI_TABLE = 4,      // table mode fp32 epilogue (see GemmProblem)
};

struct GemmClass {
  int M, N, K, count;
  int tiles_n, tiles_per_mat;
  int tile_begin;
  // Output 0 / output 1 / aux input: element pointers to matrix 0 of the class,
  // batch stride and leading dimension in elements.
  void* out0;
  long long out0_bs;
  int out0_ld;
  void* out1;
  long long out1_bs;
  int out1_ld;
  const void* aux;
  long long aux_bs;
  int aux_ld;
  const float* scale;  // per matrix of the class, or nullptr (= 1)
  int tiles_per_mat2, tile_begin2;  // tiles_per_mat / tile_begin in the CTA-pair kernel's 256-row tiles
};

struct GemmParams {
  CUtensorMap mapA[kMaxClasses];
  CUtensorMap mapB[kMaxClasses];
  GemmClass cls[kMaxClasses];
  int nclasses;
  int total_tiles;   // the tiles of the kernel launched (one-CTA or CTA-pair numbering)
  int total_tiles1, total_tiles2;  // 128 x 256 one-CTA tiles, 256 x 256 pair tiles
  float alpha, beta, gamma;
  DevStatus* status;
};

// Table mode: one entry per problem (device memory, 64-byte aligned maps).
struct GemmProblem {
  const CUtensorMap* mapA[3];  // the three bf16 planes of A and of B
  const CUtensorMap* mapB[3];
  float* out;                  // M x N fp32 (ld_out), or nullptr
  __nv_bfloat16* out_p[3];     // three-plane split of the result (ld_outp), or nullptr
  const float* aux;            // M x N fp32 (ld_aux), or nullptr; may equal out
  const int* flag;             // nullptr, or skip this problem when *flag == 0
  int M, N, K;
  int m_off, n_off;            // operand coordinates of output row/column 0 (sub-block views)
  int k_off;                   // operand coordinate of K index 0 (a K slice; multiple of 8 for K-major operands)
  int ld_out, ld_aux, ld_outp;
  int tiles_n, tile_begin;      // tiles_n: column tiles of the one-CTA kernel (128 or 256 wide)
  int tiles_n2;                 // column tiles of the CTA-pair kernel (128 wide)
  float alpha, beta;
  // Alternate destination chosen on the device: when sel != nullptr and *sel == 0
  // the result goes to out2 / out2_p (leading dimensions ld_out2 / ld_out2p) instead.
  const int* sel;
  float* out2;
  __nv_bfloat16* out2_p[3];
  int ld_out2, ld_out2p;
  int tile_begin2;             // first tile in the CTA-pair numbering (256-row tiles)
  // Update statistics (nullptr = none): for every block of 32 output rows by 64
  // columns, (sum of (out - aux)^2, number of non-finite out) is written to
  // upd[(row / 32) * ceil(N / 64) + col / 64] by the one warp that stores that block.
  float2* upd;
};

struct GemmTableParams {
  const GemmProblem* probs;
  int nprob;
  int total_tiles;   // 128-row tiles (one CTA each), or 256-row tiles for the CTA-pair kernel
  DevStatus* status;
  // nullptr, or a flag that is 0 when every problem of the launch is gated off: the
  // launch then returns before any setup
  const int* any;
  // nullptr, or two counters (profiling): the work (multiply-adds x 2) of the tiles
  // the kernel computed, and the tensor-core operations it issued
  unsigned long long* work;
};

// PA / PB: bf16 planes held per operand (SPLIT3 kinds only; 1 = a plain bf16
// operand, exact in one plane).  The products taken are the pairs (i, j), i < PA,
// j < PB, with i + j <= max(PA, PB) - 1: all six terms at or above the fp32 unit
// roundoff for (3, 3), x_i y_0 for (3, 1), the single exact product for (1, 1).
template <int KIND, int A_MN, int B_MN, int PA = (KIND == OP_BF16 ? 1 : 3), int PB = PA>
struct GemmCfg {
  static constexpr int BM = 128;
  // 128 x 256 tiles for one-plane operands (bf16 x bf16: one product per k-step, so the
  // operand stream per multiply-add is the limit and wider tiles halve it per output)
  static constexpr int BN = (KIND == OP_BF16 || (PA == 1 && PB == 1)) ? 256 : 128;
  static constexpr int ESIZE = 2;                      // bf16 planes
  static constexpr int BK = 64;                        // elements per 128-byte row
  static constexpr int UMMA_K = 16;                    // 32 bytes of K per MMA
  static constexpr int A_TILE = BM * 128;              // bytes per plane
  static constexpr int B_TILE = BN * 128;
  static constexpr int STAGE_BYTES = PA * A_TILE + PB * B_TILE;
  static constexpr int STAGES_FIT = (200 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = (KIND == OP_BF16) ? 4 : (STAGES_FIT > 6 ? 6 : STAGES_FIT);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
  static constexpr int PMAX = (PA > PB ? PA : PB) - 1;  // largest i + j taken
  static constexpr bool CORR = (PA > 1 || PB > 1);       // any cross product
  static constexpr int ACC_COLS = CORR ? 2 * BN : BN;    // main (+ correction) accumulator
  // SPLIT3: k-blocks per TMEM accumulation item.  The tensor core's accumulation
  // truncates; products with a three-plane operand fold every 2 k-blocks (8
  // truncating adds of 16 of K: within twice an fp32 evaluation's error, where
  // 16 adds were not), bf16 x bf16 every 4.  A fold per k-block costs 8 % of the
  // SOAP step: the epilogue's TMEM reads then no longer hide behind the MMAs.
  static constexpr int KCH = CORR ? 2 : 4;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;         // double-buffered
  static constexpr uint32_t IDESC = make_idesc(1u, A_MN, B_MN, BM, BN);
  static constexpr int THREADS = 320;        // producer, MMA issuer, 8 epilogue warps
  static constexpr int TABLE_THREADS = 320;
};

// Descriptor of one operand tile (rows = MN extent R, K extent = BK) at smem
// address `base`, advanced to MMA k-step `k`.
template <int MN_MAJOR, int R, int ESIZE>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int k) {
  constexpr int UMMA_K_BYTES = 32;
  if constexpr (!MN_MAJOR) {
    // K-major: rows of 128 B; the k-th 32-byte slice of every row.
    return smem_desc_sw128(base + k * UMMA_K_BYTES, 16, 1024);
  } else {
    // MN-major: the tile is R/(128/ESIZE) chunks of [BK rows x 128 B], each chunk
    // BK*128 bytes; a k-step covers UMMA_K K-rows = (32/ESIZE) rows of 128 B.
    constexpr int BK = 128 / ESIZE;
    constexpr int ROWS_PER_STEP = UMMA_K_BYTES / ESIZE;
    return smem_desc_sw128(base + k * ROWS_PER_STEP * 128, BK * 128, 1024);
  }
}

// Issue the TMA loads of one operand tile (one plane).  K-major tiles of R rows
// are loaded as R / BOXR boxes of BOXR rows (the descriptor's box height); the
// boxes land back to back, which is the same layout as one R-row box.
template <int MN_MAJOR, int R, int ESIZE, int BOXR = R>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int k0,
                                             int mn0, int b) {
  if constexpr (!MN_MAJOR) {
#pragma unroll
    for (int i = 0; i < R / BOXR; ++i) tma_load_3d(dst + i * BOXR * 128, map, bar, k0, mn0 + i * BOXR, b);
  } else {
    constexpr int CHUNK = 128 / ESIZE;  // MN elements per 128-byte row
    constexpr int BK = 128 / ESIZE;
#pragma unroll
    for (int c = 0; c < R / CHUNK; ++c) tma_load_3d(dst + c * BK * 128, map, bar, mn0 + c * CHUNK, k0, b);
  }
}

// 256-bit global stores: a lane writes one whole 32-byte sector per instruction
// (16-byte stores leave each sector half written twice, and the L1 sends both
// halves to L2 as separate partial-sector writes).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// 32 consecutive fp32 (16-byte aligned; whole sectors when 32-byte aligned)
__device__ __forceinline__ void store_f32x32(float* dst, const float* v) {
  if (aligned32(dst)) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = __float_as_uint(v[j + e]);
      st_global_v8(dst + j, w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  }
}

// 32 consecutive bf16 packed in pairs (16-byte aligned; whole sectors when 32-byte
// aligned)
__device__ __forceinline__ void store_bf16x32_packed(__nv_bfloat16* dst, const uint32_t* w) {
  if (aligned32(dst)) {
    st_global_v8(dst, w);
    st_global_v8(dst + 16, w + 8);
  } else {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int j = 0; j < 4; ++j) d[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

// 32 consecutive bf16, rounded to nearest (16-byte aligned; whole sectors when
// 32-byte aligned)
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint32_t w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    w[j] = *reinterpret_cast<uint32_t*>(&h);
  }
  if (aligned32(dst)) {
    st_global_v8(dst, w);
    st_global_v8(dst + 16, w + 8);
  } else {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int j = 0; j < 4; ++j) d[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float* v) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 q = s[j];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h[e]);
      v[8 * j + 2 * e] = f.x;
      v[8 * j + 2 * e + 1] = f.y;
    }
  }
}

// What one tile needs from its problem description.
struct TileInfo {
  const CUtensorMap* mapA[3];
  const CUtensorMap* mapB[3];
  int idx;     // class (class mode) or problem (table mode)
  int b;       // batch index inside the class (class mode), 0 in table mode
  int m0, n0;
  int K;
  bool valid;  // false: the tile's problem is gated off
  int am, bn;  // operand coordinate offsets along M (A) and N (B)
  int ko;      // operand coordinate offset along K
};

// bf16 tensor-core products per multiply-add of a (PA, PB)-plane product
template <int PA, int PB>
constexpr int kTileProducts = (PA == 3 && PB == 3) ? 6 : (PA == 1 && PB == 1) ? 1 : 3;

// ------------------------------------------------------------------ class mode
struct ClassSource {
  const GemmParams& p;
  __device__ explicit ClassSource(const GemmParams& p_) : p(p_) {}
  __device__ bool skip_all() const { return false; }
  __device__ void prefetch_aux(const TileInfo&, int, int, int) const {}
  template <int PRODUCTS>
  __device__ void count_work(const TileInfo&, int, int) const {}
  __device__ int total_tiles() const { return p.total_tiles; }
  __device__ DevStatus* status() const { return p.status; }
  __device__ void prefetch() const {
    for (int c = 0; c < p.nclasses; ++c) {
      tma_prefetch_desc(&p.mapA[c]);
      tma_prefetch_desc(&p.mapB[c]);
    }
  }
  __device__ TileInfo decode(int tile, int BM, int BN) const {
    const bool pair = BM == 256;
    int c = 0;
#pragma unroll 1
    while (c + 1 < p.nclasses && tile >= (pair ? p.cls[c + 1].tile_begin2 : p.cls[c + 1].tile_begin)) ++c;
    const GemmClass& C = p.cls[c];
    const int local = tile - (pair ? C.tile_begin2 : C.tile_begin);
    const int tpm = pair ? C.tiles_per_mat2 : C.tiles_per_mat;
    const int b = local / tpm;
    const int r = local - b * tpm;
    TileInfo t;
    t.mapA[0] = &p.mapA[c];
    t.mapB[0] = &p.mapB[c];
    t.mapA[1] = t.mapA[2] = t.mapB[1] = t.mapB[2] = nullptr;
    t.idx = c;
    t.b = b;
    t.m0 = (r / C.tiles_n) * BM;
    t.n0 = (r % C.tiles_n) * BN;
    t.K = C.K;
    t.valid = true;
    t.am = 0;
    t.bn = 0;
    t.ko = 0;
    return t;
  }
  __device__ int cols(const TileInfo& t) const { return p.cls[t.idx].N; }

  // Epilogue for 32 consecutive columns [col0, col0+32) of one tile row.
  template <int EPI>
  __device__ __forceinline__ void epilogue(const TileInfo& t, int row, int col0, float* v) const {
    const GemmClass& C = p.cls[t.idx];
    const int b = t.b;
    if (row >= C.M) return;
    const bool full = (col0 + 32 <= C.N);
    if constexpr (EPI == EPI_STORE_F32) {
      float* out =
          reinterpret_cast<float*>(C.out0) + (long long)b * C.out0_bs + (long long)row * C.out0_ld + col0;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(out + j) =
              make_float4(p.alpha * v[j], p.alpha * v[j + 1], p.alpha * v[j + 2], p.alpha * v[j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < C.N) out[j] = p.alpha * v[j];
      }
    } else {
      const float s = C.scale ? C.scale[b] : 1.0f;
      if constexpr (EPI == EPI_GRAM) {
        const float s2 = s * s;
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= s2;
      } else {
        float a[32];
        const __nv_bfloat16* aux = reinterpret_cast<const __nv_bfloat16*>(C.aux) + (long long)b * C.aux_bs +
                                   (long long)row * C.aux_ld + col0;
        if (full) {
          load_bf16x32(aux, a);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = (col0 + j < C.N) ? __bfloat162float(aux[j]) : 0.0f;
        }
        if constexpr (EPI == EPI_POLY) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = p.beta * a[j] + p.gamma * v[j];
        } else {  // EPI_AXPY_T
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = s * (p.alpha * a[j] + v[j]);
        }
      }
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(C.out0) + (long long)b * C.out0_bs +
                           (long long)row * C.out0_ld + col0;
      if (full) {
        store_bf16x32(out, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < C.N) out[j] = __float2bfloat16_rn(v[j]);
      }
      if constexpr (EPI == EPI_AXPY_T) {
        if (C.out1 != nullptr) {
          // optional transposed copy: for each column j, the 32 lanes (consecutive
          // rows) write 32 consecutive elements of row (col0 + j) of out1.
          __nv_bfloat16* tp = reinterpret_cast<__nv_bfloat16*>(C.out1) + (long long)b * C.out1_bs + row;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < C.N) tp[(long long)(col0 + j) * C.out1_ld] = __float2bfloat16_rn(v[j]);
        }
      }
    }
  }
};

// ------------------------------------------------------------------ table mode
struct TableSource {
  const GemmTableParams& p;
  __device__ explicit TableSource(const GemmTableParams& p_) : p(p_) {}
  __device__ bool skip_all() const { return p.any != nullptr && *p.any == 0; }
  // L2 prefetch of the aux row segment [col0, col0 + cols) the epilogue thread of `row`
  // will read, issued before the tile's K loop so that the reads after it hit L2.
  __device__ __forceinline__ void prefetch_aux(const TileInfo& t, int row, int col0, int cols) const {
    const GemmProblem& P = p.probs[t.idx];
    if (P.aux == nullptr || row >= P.M) return;
    const float* a = P.aux + (long long)row * P.ld_aux;
    for (int c = col0; c < col0 + cols && c < P.N; c += 32)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a + c));
  }
  // Profiling: the work of one computed tile (called once per tile by the MMA issuer).
  template <int PRODUCTS>
  __device__ void count_work(const TileInfo& t, int BM, int BN) const {
    if (p.work == nullptr) return;
    const GemmProblem& P = p.probs[t.idx];
    const unsigned long long rows = (unsigned long long)min(BM, P.M - t.m0);
    const unsigned long long cols = (unsigned long long)min(BN, P.N - t.n0);
    const unsigned long long f = 2ull * rows * cols * (unsigned long long)t.K;
    atomicAdd(p.work, f);
    atomicAdd(p.work + 1, f * PRODUCTS);
  }
  __device__ int total_tiles() const { return p.total_tiles; }
  __device__ DevStatus* status() const { return p.status; }
  __device__ void prefetch() const {}
  __device__ TileInfo decode(int tile, int BM, int BN) const {
    const bool pair = BM == 256;
    // the staged table is followed by the problems' first tiles (one-CTA numbering, then
    // the CTA-pair numbering): a compact search instead of probing the large records
    const int* starts = reinterpret_cast<const int*>(p.probs + p.nprob) + (pair ? p.nprob : 0);
    const int lo = find_start(starts, p.nprob, tile);
    const GemmProblem& P = p.probs[lo];
    const int r = tile - (pair ? P.tile_begin2 : P.tile_begin);
    const int tn = pair ? P.tiles_n2 : P.tiles_n;
    TileInfo t;
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      t.mapA[q] = P.mapA[q];
      t.mapB[q] = P.mapB[q];
    }
    t.idx = lo;
    t.b = 0;
    t.m0 = (r / tn) * BM;
    t.n0 = (r % tn) * BN;
    t.K = P.K;
    t.valid = (P.flag == nullptr) || (*P.flag != 0);
    t.am = P.m_off;
    t.bn = P.n_off;
    t.ko = P.k_off;
    return t;
  }
  __device__ int cols(const TileInfo& t) const { return p.probs[t.idx].N; }

  // One problem's epilogue parameters, read once per tile with the device-chosen
  // destination resolved: held in registers, they are not re-read after every store
  // (the stores could alias the problem records as far as the compiler knows).
  struct Epi {
    float* out;
    __nv_bfloat16* outp[3];
    const float* aux;
    float2* upd;
    int M, N, ld_out, ld_outp, ld_aux;
    float alpha, beta;
  };
  __device__ __forceinline__ Epi epi(const TileInfo& t) const {
    const GemmProblem& P = p.probs[t.idx];
    Epi e;
    const bool alt = (P.sel != nullptr) && (*P.sel == 0);
    e.out = alt ? P.out2 : P.out;
#pragma unroll
    for (int q = 0; q < 3; ++q) e.outp[q] = alt ? P.out2_p[q] : P.out_p[q];
    e.ld_out = alt ? P.ld_out2 : P.ld_out;
    e.ld_outp = alt ? P.ld_out2p : P.ld_outp;
    e.aux = P.aux;
    e.upd = P.upd;
    e.M = P.M;
    e.N = P.N;
    e.ld_aux = P.ld_aux;
    e.alpha = P.alpha;
    e.beta = P.beta;
    return e;
  }

  // out = alpha * acc + beta * aux for 32 columns of one row; `st` accumulates the
  // update statistics (sum of (out - aux)^2, non-finite count) when the problem asks.
  __device__ __forceinline__ void epilogue_table(const Epi& e, int row, int col0, float* v, float2& st) const {
    if (row >= e.M) return;
    const bool full = (col0 + 32 <= e.N);
    if (e.aux != nullptr) {
      const float* a = e.aux + (long long)row * e.ld_aux + col0;
      const bool want = e.upd != nullptr;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 q = *reinterpret_cast<const float4*>(a + j);
          v[j] = e.alpha * v[j] + e.beta * q.x;
          v[j + 1] = e.alpha * v[j + 1] + e.beta * q.y;
          v[j + 2] = e.alpha * v[j + 2] + e.beta * q.z;
          v[j + 3] = e.alpha * v[j + 3] + e.beta * q.w;
          if (want) {
            const float d0 = v[j] - q.x, d1 = v[j + 1] - q.y, d2 = v[j + 2] - q.z, d3 = v[j + 3] - q.w;
            st.x += (d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3);
            st.y += (float)(!isfinite(v[j]) + !isfinite(v[j + 1]) + !isfinite(v[j + 2]) + !isfinite(v[j + 3]));
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (col0 + j < e.N) {
            const float old = a[j];
            v[j] = e.alpha * v[j] + e.beta * old;
            if (want) {
              const float d = v[j] - old;
              st.x += d * d;
              st.y += isfinite(v[j]) ? 0.f : 1.f;
            }
          } else {
            v[j] = 0.0f;
          }
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= e.alpha;
    }
    if (e.out != nullptr) {
      float* o = e.out + (long long)row * e.ld_out + col0;
      if (full) {
        store_f32x32(o, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < e.N) o[j] = v[j];
      }
    }
    if (e.outp[0] != nullptr) {
      // the three planes are peeled off v in place (v's last use): plane q is the
      // bf16 rounding of what the planes before it left
      const long long offp = (long long)row * e.ld_outp + col0;
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
          w[j] = *reinterpret_cast<const uint32_t*>(&h);
          const float2 f = __bfloat1622float2(h);
          v[2 * j] -= f.x;
          v[2 * j + 1] -= f.y;
        }
        __nv_bfloat16* o = e.outp[q] + offp;
        if (full) {
          store_bf16x32_packed(o, w);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < e.N)
              o[j] = __ushort_as_bfloat16((unsigned short)((j & 1) ? (w[j >> 1] >> 16) : (w[j >> 1] & 0xffffu)));
        }
      }
    }
  }

  // Warp-level reduction of the update statistics of the 32 x 64 block whose first
  // row / column are row0 / col0 (every lane of the warp calls this; fixed order).
  __device__ __forceinline__ void flush_stats(const Epi& e, int row0, int col0, float2 st, int lane) const {
    if (e.upd == nullptr) return;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      st.x += __shfl_xor_sync(0xffffffffu, st.x, o);
      st.y += __shfl_xor_sync(0xffffffffu, st.y, o);
    }
    if (lane == 0 && row0 < e.M && col0 < e.N) e.upd[(long long)(row0 >> 5) * ((e.N + 63) >> 6) + (col0 >> 6)] = st;
  }
};

// ------------------------------------------------------------------ kernel body
template <int KIND, int A_MN, int B_MN, int EPI, class Src, int PA = (KIND == OP_BF16 ? 1 : 3), int PB = PA>
__device__ __forceinline__ void gemm_body(const Src& src) {
  using Cfg = GemmCfg<KIND, A_MN, B_MN, PA, PB>;
  constexpr int BM = Cfg::BM, BN = Cfg::BN, BK = Cfg::BK, STAGES = Cfg::STAGES;
  // 8 epilogue warps, two per TMEM lane quarter, each taking half of the tile's
  // columns: twice the memory operations in flight for the epilogue's aux reads and
  // stores (and, in table mode, half the fold registers per thread).
  constexpr int EPI_WARPS = 8;
  constexpr int COLS = BN * 4 / EPI_WARPS;  // columns per epilogue warp

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ int prod_it_sh, mma_it_sh;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  DevStatus* status = src.status();
  if (src.skip_all()) return;  // uniform over the grid

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 32 * EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    prod_it_sh = 0;
    mma_it_sh = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) src.prefetch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;
  const int total = src.total_tiles();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int it = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const TileInfo t = src.decode(tile, BM, BN);
        if (!t.valid) continue;
        if constexpr (EPI == EPI_TABLE) {
#pragma unroll
          for (int q = 0; q < PA; ++q) tensormap_acquire(t.mapA[q]);
#pragma unroll
          for (int q = 0; q < PB; ++q) tensormap_acquire(t.mapB[q]);
        }
        const int nk = (t.K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty_bar[s], ph ^ 1, status, 1, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], Cfg::STAGE_BYTES);
          const int am = t.am + t.m0, bn = t.bn + t.n0, kc = t.ko + kb * BK;
          // stage layout: A planes, then B planes
#pragma unroll
          for (int q = 0; q < PA; ++q)
            load_operand<A_MN, BM, Cfg::ESIZE>(st + q * Cfg::A_TILE, t.mapA[q], &full_bar[s], kc, am, t.b);
#pragma unroll
          for (int q = 0; q < PB; ++q)
            load_operand<B_MN, BN, Cfg::ESIZE, (EPI == EPI_TABLE ? 64 : 128)>(
                st + PA * Cfg::A_TILE + q * Cfg::B_TILE, t.mapB[q], &full_bar[s], kc, bn, t.b);
        }
        if (!ok) break;
      }
      prod_it_sh = it;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      // One accumulation item per (tile, K-chunk): SPLIT3 accumulates KCH k-blocks
      // per item (the epilogue folds the items in fp32 registers), bf16 the whole K.
      int it = 0, used = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo t = src.decode(tile, BM, BN);
        if (!t.valid) continue;
        src.template count_work<kTileProducts<PA, PB>>(t, BM, BN);
        const int nk = (t.K + BK - 1) / BK;
        const int nch = (KIND == OP_SPLIT3) ? (nk + Cfg::KCH - 1) / Cfg::KCH : 1;
        for (int c = 0; c < nch && ok; ++c) {
          const int acc = used & 1;
          const uint32_t aph = (used >> 1) & 1;
          ++used;
          if (!mbar_wait(&tempty_bar[acc], aph ^ 1, status, 2, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_COLS;
          const int kb0 = (KIND == OP_SPLIT3) ? c * Cfg::KCH : 0;
          const int kb1 = (KIND == OP_SPLIT3) ? min(nk, kb0 + Cfg::KCH) : nk;
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&full_bar[s], ph, status, 3, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_base = smem_u32(smem + s * Cfg::STAGE_BYTES);
            const uint32_t b_base = a_base + PA * Cfg::A_TILE;
#pragma unroll
            for (int k = 0; k < BK / Cfg::UMMA_K; ++k) {
              const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
              if constexpr (KIND == OP_BF16) {
                umma_f16(d_tmem, operand_desc<A_MN, BM, Cfg::ESIZE>(a_base, k),
                         operand_desc<B_MN, BN, Cfg::ESIZE>(b_base, k), Cfg::IDESC, accum);
              } else {
                // cross products (smallest first) into the correction accumulator,
                // the main product into its own
                constexpr int pa[5] = {1, 0, 2, 0, 1};
                constexpr int pb[5] = {1, 2, 0, 1, 0};
                bool first = true;
#pragma unroll
                for (int q = 0; q < 5; ++q) {
                  if (pa[q] < PA && pb[q] < PB && pa[q] + pb[q] <= Cfg::PMAX) {
                    umma_f16(d_tmem + BN, operand_desc<A_MN, BM, Cfg::ESIZE>(a_base + pa[q] * Cfg::A_TILE, k),
                             operand_desc<B_MN, BN, Cfg::ESIZE>(b_base + pb[q] * Cfg::B_TILE, k), Cfg::IDESC,
                             first ? accum : 1u);
                    first = false;
                  }
                }
                umma_f16(d_tmem, operand_desc<A_MN, BM, Cfg::ESIZE>(a_base, k),
                         operand_desc<B_MN, BN, Cfg::ESIZE>(b_base, k), Cfg::IDESC, accum);
              }
            }
            umma_commit(&empty_bar[s]);
          }
          if (!ok) break;
          umma_commit(&tfull_bar[acc]);
        }
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_it_sh = it;
      umma_commit(&drain_bar);
      mbar_wait(&drain_bar, 0, status, 5, abort_flag, false);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int cb = ((warp - 2) >> 2) * COLS;  // first column of this warp's share
    const int row_in_tile = q * 32 + lane;
    int used = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileInfo t = src.decode(tile, BM, BN);
      if (!t.valid) continue;
      const int row = t.m0 + row_in_tile;
      const int ncols = src.cols(t);
      if constexpr (KIND == OP_BF16) {
        const int acc = used & 1;
        const uint32_t aph = (used >> 1) & 1;
        ++used;
        const bool w = mbar_wait(&tfull_bar[acc], aph, status, 4, abort_flag);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS + cb;
#pragma unroll 1
        for (int ch = 0; ch < COLS / 32; ++ch) {
          uint32_t rr[32];
          tmem_ld_32x32b_x32(tacc + ch * 32, rr);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(rr[j]);
          if (t.n0 + cb + ch * 32 < ncols) src.template epilogue<EPI>(t, row, t.n0 + cb + ch * 32, v);
        }
        tc_fence_before();
        mbar_arrive_relaxed(&tempty_bar[acc]);
      } else {
        if constexpr (EPI == EPI_TABLE) src.prefetch_aux(t, row, t.n0 + cb, COLS);
        // fold the K-chunk accumulators (main + correction) into fp32 registers
        const int nk = (t.K + BK - 1) / BK;
        const int nch = (nk + Cfg::KCH - 1) / Cfg::KCH;
        float run[COLS];
#pragma unroll
        for (int j = 0; j < COLS; ++j) run[j] = 0.0f;
        for (int c = 0; c < nch; ++c) {
          const int acc = used & 1;
          const uint32_t aph = (used >> 1) & 1;
          ++used;
          const bool w = mbar_wait(&tfull_bar[acc], aph, status, 4, abort_flag);
          if (!__all_sync(0xffffffffu, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS + cb;
#pragma unroll
          for (int ch = 0; ch < COLS / 32; ++ch) {
            uint32_t rm[32];
            tmem_ld_32x32b_x32(tacc + ch * 32, rm);
            if constexpr (Cfg::CORR) {
              uint32_t rc[32];
              tmem_ld_32x32b_x32(tacc + BN + ch * 32, rc);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) run[ch * 32 + j] += __uint_as_float(rm[j]) + __uint_as_float(rc[j]);
            } else {
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) run[ch * 32 + j] += __uint_as_float(rm[j]);
            }
          }
          tc_fence_before();
          mbar_arrive_relaxed(&tempty_bar[acc]);
        }
        if (!ok) break;
        if constexpr (EPI == EPI_TABLE) {
          static_assert(COLS % 64 == 0, "update statistics are kept per 32 x 64 block");
          const auto e = src.epi(t);
#pragma unroll
          for (int h = 0; h < COLS / 64; ++h) {
            float2 st = make_float2(0.f, 0.f);
#pragma unroll
            for (int ch = 2 * h; ch < 2 * h + 2; ++ch)
              if (t.n0 + cb + ch * 32 < ncols) src.epilogue_table(e, row, t.n0 + cb + ch * 32, &run[ch * 32], st);
            src.flush_stats(e, t.m0 + q * 32, t.n0 + cb + 64 * h, st, lane);
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < COLS / 32; ++ch)
            if (t.n0 + cb + ch * 32 < ncols) src.template epilogue<EPI>(t, row, t.n0 + cb + ch * 32, &run[ch * 32]);
        }
      }
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0) {
    // after an early exit, let TMA loads still in flight land before the CTA ends
    for (int j = mma_it_sh; j < prod_it_sh; ++j)
      mbar_wait(&full_bar[j % STAGES], (j / STAGES) & 1, status, 6, abort_flag, false);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA-pair kernel body
// Table mode on a pair of CTAs (cluster of 2): the pair owns 256 x 128 output
// tiles.  CTA r loads A rows [128 r, +128) and B columns [64 r, +64) of every
// plane into its own shared memory, with the transfers counted on the first
// CTA's mbarrier; the first CTA issues tcgen05.mma.cta_group::2 (M = 256,
// N = 128), which reads both CTAs' tiles and writes each CTA's 128 accumulator
// rows into that CTA's TMEM; its commits reach both CTAs' barriers.  Each CTA's
// epilogue folds and stores its own rows and releases the accumulator on the
// first CTA's barrier.  Per 128 x 128 of output a CTA loads 3/4 of the bytes of
// the one-CTA kernel, which leaves room for a third pipeline stage.
template <int A_MN, int B_MN, int PA, int PB, int KIND = OP_SPLIT3>
struct GemmPairCfg {
  static constexpr int BM = 128;   // rows per CTA (the pair's tile has 256)
  // columns of the pair's tile: 128 for the fp32-faithful products (main and
  // correction accumulators, double-buffered, fill the tensor memory), 256 for the
  // bf16 Newton-Schulz products (one accumulator over the whole K)
  static constexpr int BN = (KIND == OP_BF16) ? 256 : 128;
  static constexpr int BNH = BN / 2;  // columns of B loaded by each CTA
  static constexpr int ESIZE = 2;
  static constexpr int BK = 64;
  static constexpr int UMMA_K = 16;
  static constexpr int A_TILE = BM * 128;
  static constexpr int B_TILE = BNH * 128;
  static constexpr int STAGE_BYTES = PA * A_TILE + PB * B_TILE;
  static constexpr int STAGES_FIT = (216 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
  static constexpr int PMAX = (PA > PB ? PA : PB) - 1;
  static constexpr bool CORR = (PA > 1 || PB > 1);
  static constexpr int ACC_COLS = CORR ? 2 * BN : BN;
  // as in the one-CTA kernel; bf16 Newton-Schulz products accumulate the whole K
  static constexpr int KCH = CORR ? 2 : (KIND == OP_BF16 ? (1 << 28) : 4);
  // the pair allocates all of TMEM, so both CTAs' accumulators start at the same
  // column (the pair MMA writes one address in both)
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC = make_idesc(1u, A_MN, B_MN, 256, BN);
  static constexpr int EPI_WARPS = 8;  // two per TMEM lane quarter, half of the columns each
  static constexpr int COLS = BN / 2;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
};

// KIND / EPI / Src: the fp32-faithful table products (OP_SPLIT3, EPI_TABLE,
// TableSource) or the bf16 Newton-Schulz class products (OP_BF16, a class epilogue,
// ClassSource; 256 x 256 pair tiles).
template <int A_MN, int B_MN, int PA, int PB, int KIND = OP_SPLIT3, int EPI = EPI_TABLE, class Src = TableSource>
__device__ __forceinline__ void gemm_body_pair(const Src& src) {
  using Cfg = GemmPairCfg<A_MN, B_MN, PA, PB, KIND>;
  constexpr int BN = Cfg::BN, BK = Cfg::BK, STAGES = Cfg::STAGES;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ int prod_it_sh, mma_it_sh;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int npairs = gridDim.x >> 1;
  const int pair_id = blockIdx.x >> 1;
  DevStatus* status = src.status();
  // uniform over the grid: both CTAs of a pair leave before any cluster operation
  if (src.skip_all()) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 2 * 32 * Cfg::EPI_WARPS);  // both CTAs' epilogue threads (first CTA's barrier)
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    prod_it_sh = 0;
    mma_it_sh = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;
  const int total = src.total_tiles();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      int it = 0;
      for (int tile = pair_id; tile < total; tile += npairs) {
        const TileInfo t = src.decode(tile, 256, BN);
        if (!t.valid) continue;
        if constexpr (EPI == EPI_TABLE) {  // table descriptors live in global memory
#pragma unroll
          for (int q = 0; q < PA; ++q) tensormap_acquire(t.mapA[q]);
#pragma unroll
          for (int q = 0; q < PB; ++q) tensormap_acquire(t.mapB[q]);
        }
        const int nk = (t.K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty_bar[s], ph ^ 1, status, 11, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          if (leader) mbar_arrive_expect_tx(&full_bar[s], 2 * Cfg::STAGE_BYTES);
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[s]), 0);
          const int am = t.am + t.m0 + 128 * (int)rank, bn = t.bn + t.n0 + Cfg::BNH * (int)rank;
          const int kc = t.ko + kb * BK;
#pragma unroll
          for (int q = 0; q < PA; ++q) {
            uint8_t* dst = st + q * Cfg::A_TILE;
            if constexpr (!A_MN) {
              tma_load_3d_pair(dst, t.mapA[q], fb, kc, am, t.b);
            } else {
#pragma unroll
              for (int c = 0; c < 128 / 64; ++c)
                tma_load_3d_pair(dst + c * BK * 128, t.mapA[q], fb, am + c * 64, kc, t.b);
            }
          }
#pragma unroll
          for (int q = 0; q < PB; ++q) {
            uint8_t* dst = st + PA * Cfg::A_TILE + q * Cfg::B_TILE;
            if constexpr (!B_MN) {
              tma_load_3d_pair(dst, t.mapB[q], fb, kc, bn, t.b);  // one box of BNH rows
            } else {
#pragma unroll
              for (int c = 0; c < Cfg::BNH / 64; ++c)
                tma_load_3d_pair(dst + c * BK * 128, t.mapB[q], fb, bn + c * 64, kc, t.b);
            }
          }
        }
        if (!ok) break;
      }
      prod_it_sh = it;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (first CTA)
      int it = 0, used = 0;
      bool ok = true;
      for (int tile = pair_id; tile < total && ok; tile += npairs) {
        const TileInfo t = src.decode(tile, 256, BN);
        if (!t.valid) continue;
        src.template count_work<kTileProducts<PA, PB>>(t, 256, BN);
        const int nk = (t.K + BK - 1) / BK;
        const int nch = (nk + Cfg::KCH - 1) / Cfg::KCH;
        for (int c = 0; c < nch && ok; ++c) {
          const int acc = used & 1;
          const uint32_t aph = (used >> 1) & 1;
          ++used;
          if (!mbar_wait(&tempty_bar[acc], aph ^ 1, status, 12, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_COLS;
          const int kb0 = c * Cfg::KCH;
          const int kb1 = min(nk, kb0 + Cfg::KCH);
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&full_bar[s], ph, status, 13, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_base = smem_u32(smem + s * Cfg::STAGE_BYTES);
            const uint32_t b_base = a_base + PA * Cfg::A_TILE;
#pragma unroll
            for (int k = 0; k < BK / Cfg::UMMA_K; ++k) {
              const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
              constexpr int pa[5] = {1, 0, 2, 0, 1};
              constexpr int pb[5] = {1, 2, 0, 1, 0};
              bool first = true;
#pragma unroll
              for (int q = 0; q < 5; ++q) {
                if (pa[q] < PA && pb[q] < PB && pa[q] + pb[q] <= Cfg::PMAX) {
                  umma_f16_pair(d_tmem + BN, operand_desc<A_MN, 128, 2>(a_base + pa[q] * Cfg::A_TILE, k),
                                operand_desc<B_MN, Cfg::BNH, 2>(b_base + pb[q] * Cfg::B_TILE, k), Cfg::IDESC,
                                first ? accum : 1u);
                  first = false;
                }
              }
              umma_f16_pair(d_tmem, operand_desc<A_MN, 128, 2>(a_base, k), operand_desc<B_MN, Cfg::BNH, 2>(b_base, k),
                            Cfg::IDESC, accum);
            }
            umma_commit_pair(&empty_bar[s], 0x3);
          }
          if (!ok) break;
          umma_commit_pair(&tfull_bar[acc], 0x3);
        }
      }
      mma_it_sh = it;
      umma_commit_pair(&drain_bar, 0x3);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    constexpr int COLS = Cfg::COLS;
    const int q = warp & 3;
    const int cb = ((warp - 2) >> 2) * COLS;
    const int row_in_tile = q * 32 + lane;
    const uint32_t tempty_lead[2] = {mapa_shared(smem_u32(&tempty_bar[0]), 0), mapa_shared(smem_u32(&tempty_bar[1]), 0)};
    int used = 0;
    bool ok = true;
    for (int tile = pair_id; tile < total && ok; tile += npairs) {
      const TileInfo t = src.decode(tile, 256, BN);
      if (!t.valid) continue;
      const int row = t.m0 + 128 * (int)rank + row_in_tile;
      const int ncols = src.cols(t);
      if constexpr (EPI != EPI_TABLE) {
        // bf16 class products: one accumulation item per tile, stored chunk by chunk
        const int acc = used & 1;
        const uint32_t aph = (used >> 1) & 1;
        ++used;
        const bool w = mbar_wait(&tfull_bar[acc], aph, status, 14, abort_flag);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS + cb;
#pragma unroll 1
        for (int ch = 0; ch < COLS / 32; ++ch) {
          uint32_t rr[32];
          tmem_ld_32x32b_x32(tacc + ch * 32, rr);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(rr[j]);
          if (t.n0 + cb + ch * 32 < ncols) src.template epilogue<EPI>(t, row, t.n0 + cb + ch * 32, v);
        }
        tc_fence_before();
        mbar_arrive_cluster_relaxed(tempty_lead[acc]);
        continue;
      } else {
      src.prefetch_aux(t, row, t.n0 + cb, COLS);
      const int nk = (t.K + BK - 1) / BK;
      const int nch = (nk + Cfg::KCH - 1) / Cfg::KCH;
      float run[COLS];
#pragma unroll
      for (int j = 0; j < COLS; ++j) run[j] = 0.0f;
      for (int c = 0; c < nch; ++c) {
        const int acc = used & 1;
        const uint32_t aph = (used >> 1) & 1;
        ++used;
        const bool w = mbar_wait(&tfull_bar[acc], aph, status, 14, abort_flag);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS + cb;
#pragma unroll
        for (int ch = 0; ch < COLS / 32; ++ch) {
          uint32_t rm[32];
          tmem_ld_32x32b_x32(tacc + ch * 32, rm);
          if constexpr (Cfg::CORR) {
            uint32_t rc[32];
            tmem_ld_32x32b_x32(tacc + BN + ch * 32, rc);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) run[ch * 32 + j] += __uint_as_float(rm[j]) + __uint_as_float(rc[j]);
          } else {
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) run[ch * 32 + j] += __uint_as_float(rm[j]);
          }
        }
        tc_fence_before();
        mbar_arrive_cluster_relaxed(tempty_lead[acc]);
      }
      if (!ok) break;
      static_assert(COLS % 64 == 0, "update statistics are kept per 32 x 64 block");
      const auto e = src.epi(t);
#pragma unroll
      for (int h = 0; h < COLS / 64; ++h) {
        float2 st = make_float2(0.f, 0.f);
#pragma unroll
        for (int ch = 2 * h; ch < 2 * h + 2; ++ch)
          if (t.n0 + cb + ch * 32 < ncols) src.epilogue_table(e, row, t.n0 + cb + ch * 32, &run[ch * 32], st);
        src.flush_stats(e, t.m0 + 128 * (int)rank + q * 32, t.n0 + cb + 64 * h, st, lane);
      }
      }  // table products
    }
  }

  // ---------------------------------------------------------------- teardown
  // MMAs issued by the first CTA write both CTAs' TMEM: each CTA waits for the
  // first CTA's final commit before releasing TMEM.  After an early exit the first
  // CTA lets the loads still in flight land (its full barriers count both CTAs'
  // bytes; neither producer runs more than STAGES loads ahead of the MMAs).
  if (warp == 1 && lane == 0) mbar_wait(&drain_bar, 0, status, 15, abort_flag, false);
  __syncthreads();
  if (leader && warp == 0 && lane == 0) {
    const int last = max(prod_it_sh, mma_it_sh + (*abort_flag ? STAGES : 0));
    for (int j = mma_it_sh; j < last; ++j)
      mbar_wait(&full_bar[j % STAGES], (j / STAGES) & 1, status, 16, abort_flag, false);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

template <int A_MN, int B_MN, int PA, int PB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    gemm_tc_pair_kernel(const __grid_constant__ GemmTableParams p) {
  TableSource src(p);
  gemm_body_pair<A_MN, B_MN, PA, PB>(src);
}

template <int A_MN, int B_MN, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    gemm_tc_pair_class_kernel(const __grid_constant__ GemmParams p) {
  ClassSource src(p);
  gemm_body_pair<A_MN, B_MN, 1, 1, OP_BF16, EPI, ClassSource>(src);
}

template <int KIND, int A_MN, int B_MN, int EPI>
__global__ void __launch_bounds__(320, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  ClassSource src(p);
  gemm_body<KIND, A_MN, B_MN, EPI>(src);
}

template <int A_MN, int B_MN, int PA, int PB>
__global__ void __launch_bounds__(320, 1) gemm_tc_table_kernel(const __grid_constant__ GemmTableParams p) {
  TableSource src(p);
  gemm_body<OP_SPLIT3, A_MN, B_MN, EPI_TABLE, TableSource, PA, PB>(src);
}

}  // namespace mao
