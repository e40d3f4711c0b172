// la_tc.cu -- chunkwise causal linear attention forward on the sm_100a tensor
// cores (tcgen05 + TMA + TMEM), bf16 inputs, fp32 accumulation and state.
//
// The method: "1.6 长上下文与高效注意力", section 线性注意力 (state S_t = gamma S_{t-1}
// + v_t phi(k_t)^T, output o_t = S_t phi(q_t), optional normaliser z_t), run in
// chunk mode ("Triton fused linear attention kernels", hotdry blog: chunk-mode
// forward).  Unrolling the recurrence over a chunk of C' <= C tokens that
// starts from state S_p gives, for i, j < C':
//   o_i   = gamma^(i+1) S_p qh_i + sum_{j<=i} gamma^(i-j) (qh_i . kh_j) v_j
//   den_i = gamma^(i+1) z_p . qh_i + sum_{j<=i} gamma^(i-j) (qh_i . kh_j)
//   S'    = gamma^C' S_p + sum_j gamma^(C'-1-j) v_j kh_j^T,   z' likewise.
// With the decayed keys kd_j = gamma^(C'-1-j) kh_j every decay factor becomes
// a per-row factor: multiplying o_i by gamma^(C'-1-i),
//   o_i gamma^(C'-1-i)   = qh_i (gamma^C' S_p)^T + sum_{j<=i} (qh_i . kd_j) v_j
//   den_i gamma^(C'-1-i) = qh_i . (gamma^C' z_p) + sum_{j<=i} (qh_i . kd_j),
// so one accumulator O = qh Sb^T + P V, with Sb = gamma^C' S_p (bf16) and
// P = tril(qh kd^T) (bf16, no per-element scaling), gives o_i = O_i / den'_i
// when normalised and o_i = O_i / gamma^(C'-1-i) otherwise.  This needs
// gamma^(C-1) well inside the normal range.  The other form ("value-decay
// mode") keeps phi(k) undecayed, moves the state decay onto a separate tile of
// decayed values vd_j = gamma^(C'-1-j) v_j (U = kh^T vd), takes
// P_ij = (qh_i.kh_j) gamma^(i-j) from a table, and uses two accumulators
// O_inter = qh S_p^T and O_intra = P V combined as o_i = gamma^(i+1) O_inter_i +
// O_intra_i.  It runs for heads with gamma^(C-1) < 2^-64 and always at
// d_k = 256, where it transforms the 8 KB value slice instead of the 32 KB key
// tile per chunk.
//
// One CTA owns one (sequence, head, slice of DVT value columns) and walks its
// chunks in order; the fp32 state S^T[:, slice] lives in the registers of the
// state warpgroup (d_k = 128: DVT = 128; d_k = 256: DVT = 64, so that each of
// the 128 state threads holds 128 values either way):
//   warp 0      TMA producer: Q, K, V chunk tiles into an NS-deep ring.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 2-3   transform: phi(q) and the decayed keys, in place.
//   warps 4-7   state: S <- gamma^C' S + U (U from tensor memory), the bf16
//               operand Sb for the next chunk, and the final state.
//   warps 8-11  output: score tile -> P (one chunk ahead, in tensor memory),
//               then the epilogue (row factor, cast, store) of the previous chunk.
// Per chunk, four MMAs:
//   M1  A = qh kd^T          (M=C, N=C,   K=d_k)     -> A[c%2]
//   M4  U = kd^T V           (M=128 per d_k block, N=DVT, K=C)  [value decay: kh^T vd]
//   M2  O = qh Sb^T          (M=C, N=DVT, K=d_k)     [skipped on chunk 0]
//   M3  O += P V             (M=C, N=DVT, K=C)       -> O[c%2]; P (bf16) is read from
//                            tensor memory, where the output warps wrote it over A[c%2]
//
// Every wait is bounded: on a timeout the CTA raises an abort flag, records
// the failure in a device error word, drains and frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "la_common.cuh"
#include "la_internal.h"
#include "la_sm100.cuh"
#include "la_tc_sync.cuh"

namespace la {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B, T, H, D] bf16 view as a 4-D TMA map with dims (D, H, T, B) and a
// (64, 1, C, 1) box, 128-byte swizzle: one box is a [C rows x 64 cols] slab.
bool make_map(CUtensorMap *m, const TensorView &t, int64_t B, int64_t T, int64_t H, int64_t D, int C) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)t.sh * 2, (cuuint64_t)t.st * 2, (cuuint64_t)t.sb * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  if (B == 1) strides[2] = (cuuint64_t)T * t.st * 2 > 0 ? ((cuuint64_t)T * t.st * 2 + 15) / 16 * 16 : 16;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(t.data), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

__device__ unsigned int g_tc_error = 0;
// First wait that gave up: 0x80000000 | chunk << 8 | barrier index.
__device__ unsigned int g_tc_where = 0;

namespace {

using namespace sm100;
using namespace tcsync;

constexpr int kThreads = 384;
constexpr float kSmallGammaLimit = 5.421010862427522e-20f;  // 2^-64: below, value-decay mode

struct TcArgs {
  void *out;
  int64_t o_sb, o_st, o_sh;
  const float *gamma;
  const int32_t *cu_seqlens;
  float *final_state;
  float *final_z;  // NULL, or z after each sequence's last token (normalised only)
  int64_t T;
  int H, dk, dv, phi, normalize;  // dk: the key head dim (64 in the d_k = 128 layout is zero padded)
  // Segmentation of long sequences (G = 1: none).  A sequence is split into G
  // segments of segC chunks.  The state pass (MODE 1, Gp = G - 1 CTAs per unit)
  // writes each segment's end state from a zero start to ws_s / ws_z; a scan
  // turns slot g - 1 into the start state of segment g; the output pass (MODE 0,
  // Gp = G) seeds segment g >= 1 with it.
  int G, Gp, segC;
  float *ws_s;  // [units][G-1][DK][DVT] (S^T rows)
  float *ws_z;  // [units][G-1][DK]
  float *ws_g;  // [units][G-1]: log decay of each segment (data-dependent decay)
  // Data-dependent decay: log alpha per token and head, [B * T][H] (NULL: gamma)
  const float *g;
  // Packed batches: sequence of each rank, longest first (NULL: natural order)
  const int32_t *order;
  // Output norm and gate (NG): weights [DVT], gate [B, T, H, DVT] bf16 with element strides, eps
  const float *ng_w;
  const void *ng_gate;
  int64_t ng_sb, ng_st, ng_sh;
  float ng_eps;
  // Backward epilogue: the row x of ex (bf16, element strides) at each output row's token:
  // edg[token][h] += esign * phi(x) . o (fp32 o, before rounding) when edg is set, and
  // the row written is o * phi'(x) with edphi.  ex NULL: off.
  const void *ex;
  int64_t ex_sb, ex_st, ex_sh;
  float *edg;
  float esign;
  int ephi, edphi;
  // Normalised: den_t per (token, head), [B * T][H] fp32, written by the first value
  // slice's epilogue (NULL: not written).
  float *den_out;
};

template <int DK, int DVT, int C, int NS>
struct Cfg {
  static constexpr int KB = DK / 64;    // 64-column slabs of a q/k tile
  static constexpr int VB = DVT / 64;   // 64-column slabs of a v tile
  static constexpr int MB = DK / 128;   // 128-row blocks of the state
  static constexpr int SLAB = C * 128;  // bytes of one [C rows x 64 bf16] slab
  static constexpr int QK_BYTES = KB * SLAB;
  static constexpr int V_BYTES = VB * SLAB;
  static constexpr int STAGE_BYTES = 2 * QK_BYTES + V_BYTES;
  static constexpr int SB_SLAB = DK * 128;         // [DK rows x 64 cols] bf16
  static constexpr int SB_BYTES = VB * SB_SLAB;

  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_VD = NS * STAGE_BYTES;  // decayed values (value-decay mode)
  static constexpr int OFF_SB = OFF_VD + V_BYTES;
  static constexpr int OFF_Z = OFF_SB + SB_BYTES;  // normaliser key sums z, two buffers of DK floats
  static constexpr int OFF_KSUM = OFF_Z + 2 * DK * 4;  // per stage, per transform warp: chunk key column sums
  // data-dependent decay, per stage: b_i = sum_{t<=i} log alpha_t over the chunk, i < C, and b_last at [C]
  static constexpr int OFF_DT = OFF_KSUM + NS * 2 * DK * 4;
  static constexpr int DT_STRIDE = C + 4;
  static constexpr int OFF_NGW = OFF_DT + NS * DT_STRIDE * 4;  // output-norm weights [DVT]
  static constexpr int OFF_PW = OFF_NGW + DVT * 4;
  static constexpr int OFF_BAR = OFF_PW + ((C + 1) * 4 + 15) / 16 * 16;
  // barriers
  static constexpr int B_FULL = 0, B_EMPTY = NS, B_XFORM = 2 * NS, B_AFULL = 3 * NS, B_PFULL = 3 * NS + 2,
                       B_UFULL = 3 * NS + 4, B_UEMPTY = 3 * NS + 5, B_SBFULL = 3 * NS + 6, B_SBEMPTY = 3 * NS + 7,
                       B_OFULL = 3 * NS + 8, B_OEMPTY = 3 * NS + 10, B_ZFULL = 3 * NS + 12, NBAR = 3 * NS + 14;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_USED = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment

  // tensor memory columns
  static constexpr int T_U = 0;                // per-chunk state update: MB blocks of DVT columns
  static constexpr int T_A = MB * DVT;         // two score tiles of C columns
  static constexpr int T_O = T_A + 2 * C;      // output tiles of DVT columns (below)
  // Decayed-key mode double-buffers one accumulator per chunk: O[b] at T_O +
  // b DVT.  Value-decay mode needs two (inter, intra); they are double-buffered
  // too (pair b at T_O + 2 b DVT) when four tiles fit, else one pair is reused.
  static constexpr bool VD_DB = T_O + 4 * DVT <= 512;
  static constexpr int T_COLS_USED = T_O + (VD_DB ? 4 : 2) * DVT;
  static constexpr int T_COLS = T_COLS_USED <= 32 ? 32 : T_COLS_USED <= 64 ? 64 : T_COLS_USED <= 128 ? 128
                                : T_COLS_USED <= 256 ? 256 : 512;
  static constexpr int RPT = MB * DVT;  // state values held per state-warpgroup thread

  static_assert(C == 64, "score tiles use the M=64 tensor-memory layout");
  static_assert(DK % 128 == 0 && DVT % 64 == 0, "tile shape");
  static_assert(RPT <= 128, "state registers");
  static_assert(T_COLS_USED <= 512, "tensor memory");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// phi for the bf16 tensor-core operands: elu(x) + 1, with e^x = 2^(x log2 e)
// on the PTX ex2.approx.ftz instruction (one multiply and one special-function
// op; relative error ~2^-22, far below the bf16 rounding (2^-9) the operand
// gets right after).  Branch-free: the exponential is taken for every lane (of
// min(x, 0), so it cannot overflow) and the result is a select.
__device__ __forceinline__ float phi_fast(float x) {
  constexpr float kLog2e = 1.4426950408889634f;
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(fminf(x, 0.f) * kLog2e));
  return x > 0.f ? x + 1.f : e;
}

// swish(g) = g sigmoid(g) with sigmoid(g) = (1 + tanh(g / 2)) / 2 on the PTX
// tanh.approx instruction: one special-function op per element (relative
// error ~2^-11, below the bf16 rounding of the output).
__device__ __forceinline__ float swish_fast(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return x * fmaf(0.5f, t, 0.5f);
}

// Transform of one [C x 64k] tile by the 64 transform threads (bf16 in and out):
// with STORE, dst = wv[row] * (FEAT ? phi(src) : src); with SUM, also the column
// sums sum_rows wsum[row] * (FEAT ? phi(src) : src), one fp32 [64k] row per warp
// in ksum.  Thread tt owns the 16-byte vectors tt + 64 m; vector tt + 64 m sits
// in row tt/8 + 8 (m mod 8) of slab m / 8 and physical 16-byte chunk tt mod 8,
// which under the 128-byte swizzle holds the logical 8-column block
// (tt mod 8) ^ (tt/8 mod 8) in every row this thread visits.  The four lanes of
// a warp holding the same block are lane ^ 9, ^ 18, ^ 27, so two shuffle rounds
// finish the warp's sums.  Each batch keeps one slab's 8 loads in flight.
template <bool FEAT, bool STORE, bool SUM>
__device__ __forceinline__ void xform_tile(const uint8_t *src, uint8_t *dst, int tt, int nv, const float (&wv)[8],
                                           const float (&wsum)[8], float *ksum) {
#pragma unroll 1
  for (int m0 = 0; m0 < nv; m0 += 8) {
    uint4 x[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) x[m] = *reinterpret_cast<const uint4 *>(src + (tt + 64 * (m0 + m)) * 16);
    float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      float f[8];
      unpack8(x[m], f);
      if (FEAT) {
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] = phi_fast(f[u]);
      }
      if (SUM) {
#pragma unroll
        for (int u = 0; u < 8; ++u) part[u] = fmaf(wsum[m], f[u], part[u]);
      }
      if (STORE) {
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] *= wv[m];
        *reinterpret_cast<uint4 *>(dst + (tt + 64 * (m0 + m)) * 16) = pack8(f);
      }
    }
    if (SUM) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        part[u] += __shfl_xor_sync(0xffffffffu, part[u], 9);
        part[u] += __shfl_xor_sync(0xffffffffu, part[u], 18);
      }
      if ((tt & 31) < 8) {
        float *o = ksum + (m0 / 8) * 64 + (((tt & 7) ^ ((tt >> 3) & 7)) << 3);
        *reinterpret_cast<float4 *>(o) = make_float4(part[0], part[1], part[2], part[3]);
        *reinterpret_cast<float4 *>(o + 4) = make_float4(part[4], part[5], part[6], part[7]);
      }
    }
  }
}

// REV: reverse time.  The sequence is walked from its end: chunk c is the
// window of C tokens ending (C c) tokens before the end, and inside it token
// row i stands for position i' = C - 1 - i of the reversed sequence.  Every
// formula of the forward then holds in the primed indices (valid rows
// i' < C', causal j' <= i'); the tiles stay in natural row order, so the
// products need no change.  This runs the anti-causal sums of the backward
// pass (sum over i >= j) on the same kernel.  With a per-token decay the
// anti-causal weight exp(b_i - b_j), i >= j, is the product of the decays of
// tokens j+1 .. i; in reversed positions that is the forward's weight for the
// decays shifted by one token, g''(i') = g(token of i' + 1), which is what
// the transform warps load (zero for the last token of the sequence, whose
// reversed predecessor state is zero).
// NG: the output RMSNorm with a Swish gate in the epilogue (d_v == DVT).
template <int DK, int DVT, int C, int NS, bool NORM, bool ELU, int MODE, bool GATED, bool REV, bool NG = false>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const TcArgs a) {
  using G = Cfg<DK, DVT, C, NS>;
  static_assert(!(REV && NORM), "reverse time is built for the unnormalised forms");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *z = reinterpret_cast<float *>(sm + G::OFF_Z);
  float *ksum = reinterpret_cast<float *>(sm + G::OFF_KSUM);
  float *dtab = reinterpret_cast<float *>(sm + G::OFF_DT);  // [NS][DT_STRIDE]
  float *ngw = reinterpret_cast<float *>(sm + G::OFF_NGW);  // [DVT]
  float *pw = reinterpret_cast<float *>(sm + G::OFF_PW);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + G::OFF_BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + G::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + G::OFF_MISC + 4);
  const Sync sy{bars, abort_flag, &g_tc_error, &g_tc_where};

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  // elu + 1: the output warps apply phi to the query tiles (they are idle most of
  // a chunk), so the two transform warps only handle keys and values
  constexpr bool kQByOutput = ELU && MODE == 0;

  // ---- the unit this CTA owns
  // value slices; a d_v narrower than DVT (64 at d_k <= 128) runs in one slice whose
  // columns past d_v read TMA zero fill and are never written out
  const int NVT = (a.dv + DVT - 1) / DVT;
  const int unit = blockIdx.x / a.Gp;  // (sequence, head, value slice)
  const int seg = blockIdx.x % a.Gp;
  const int vt = unit % NVT;
  const int h = (unit / NVT) % a.H;
  const int n = a.order ? a.order[unit / (NVT * a.H)] : unit / (NVT * a.H);
  int64_t start, len;
  int bidx;
  if (a.cu_seqlens) {
    bidx = 0;
    start = a.cu_seqlens[n];
    len = (int64_t)a.cu_seqlens[n + 1] - start;
  } else {
    bidx = n;
    start = 0;
    len = a.T;
  }
  // natural end of the walk (reverse time): the segment starts c0 tokens before the sequence end
  int64_t rend = start + len;
  if (a.G > 1) {  // this CTA's segment of the sequence
    const int64_t c0 = (int64_t)seg * a.segC * C;
    start += c0;
    rend -= c0;
    len = max((int64_t)0, min(len - c0, (int64_t)a.segC * C));
  }
  const bool has_init = MODE == 0 && a.G > 1 && seg > 0;  // start state from the scan
  const bool last_seg = a.G == 1 || seg == a.G - 1;
  const int64_t ws_slot = (int64_t)unit * (a.G - 1) + (MODE == 1 ? seg : seg - 1);
  const int nchunks = (int)((len + C - 1) / C);
  const float g = GATED ? 1.f : a.gamma[h];

  // ---- setup
  if (tid <= C) pw[tid] = decay_pow(g, tid);
  if (NG)
    for (int i = tid; i < DVT; i += kThreads) ngw[i] = a.ng_w[i];
  // z buffer (c & 1) holds z after chunk c; buffer 1 starts with the z before chunk 0
  for (int i = tid; i < DK; i += kThreads) z[DK + i] = (NORM && has_init) ? a.ws_z[ws_slot * DK + i] : 0.f;
  if (tid == 0) {
    for (int i = 0; i < G::NBAR; ++i) {
      uint32_t cnt = 1;
      if (i >= G::B_XFORM && i < G::B_XFORM + NS)
        cnt = kQByOutput ? 64 + 128 : 64;  // transform warps (keys, values) [+ output warps (queries)]
      else if ((i >= G::B_PFULL && i < G::B_PFULL + 2) ||
          i == G::B_UEMPTY || i == G::B_SBFULL || (i >= G::B_ZFULL && i < G::B_ZFULL + 2) ||
          (i >= G::B_OEMPTY && i < G::B_OEMPTY + 2))
        cnt = 128;
      mbar_init(bars + i, cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) tmem_alloc(tmem_slot, G::T_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // value-decay mode: always with a data-dependent decay (its factors are all <= 1)
  const bool vd_mode = GATED || DK == 256 || ((g < 1.f) && (pw[C - 1] < kSmallGammaLimit));
  // output accumulators of chunk c: buffer ob(c), completion parity oph(c)
  auto out_buf = [&](int c) -> int { return (vd_mode && !G::VD_DB) ? 0 : (c & 1); };
  auto out_phase = [&](int c) -> uint32_t { return (vd_mode && !G::VD_DB) ? (c & 1) : ((c >> 1) & 1); };

  auto chunk_len = [&](int c) -> int { return (int)min((int64_t)C, len - (int64_t)c * C); };
  // first (natural) token of chunk c's window; in reverse time it may lie before
  // the sequence start (those rows are masked, or read as zeros by TMA)
  auto tok0 = [&](int c) -> int64_t { return REV ? rend - (int64_t)(c + 1) * C : start + (int64_t)c * C; };
  // row of the (reversed) sequence that tile row r stands for
  auto lrow = [&](int r) -> int { return REV ? C - 1 - r : r; };
  auto q_tile = [&](int s) { return sm + G::OFF_STAGE + s * G::STAGE_BYTES; };
  auto k_tile = [&](int s) { return sm + G::OFF_STAGE + s * G::STAGE_BYTES + G::QK_BYTES; };
  auto v_tile = [&](int s) { return sm + G::OFF_STAGE + s * G::STAGE_BYTES + 2 * G::QK_BYTES; };
  uint8_t *vd_tile = sm + G::OFF_VD;
  uint8_t *sb_tile = sm + G::OFF_SB;

  if (warp < 4) {
    reg_dealloc<104>();
    if (warp == 0 && lane == 0) {
      // ============================================================ TMA producer
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % NS, k = c / NS;
        if (!wait_bar(sy, G::B_EMPTY + s, (k & 1) ^ 1, c)) break;
        mbar_arrive_expect_tx(bars + G::B_FULL + s, MODE == 1 ? G::STAGE_BYTES - G::QK_BYTES : G::STAGE_BYTES);
        const int t0 = (int)tok0(c);
        for (int kb = 0; kb < G::KB; ++kb) {
          if (MODE == 0) tma_load_4d(q_tile(s) + kb * G::SLAB, &tm_q, bars + G::B_FULL + s, kb * 64, h, t0, bidx);
          tma_load_4d(k_tile(s) + kb * G::SLAB, &tm_k, bars + G::B_FULL + s, kb * 64, h, t0, bidx);
        }
        for (int vb = 0; vb < G::VB; ++vb)
          tma_load_4d(v_tile(s) + vb * G::SLAB, &tm_v, bars + G::B_FULL + s, vt * DVT + vb * 64, h, t0, bidx);
        issued = c + 1;
      }
      if (*abort_flag) {  // let every issued copy land before the CTA exits
        for (int c = max(0, issued - NS); c < issued; ++c) drain_bar(sy, G::B_FULL + c % NS, (c / NS) & 1);
      }
    } else if (warp == 1 && lane == 0) {
      // ============================================================ MMA issuer
      constexpr uint32_t ID_M1 = idesc_bf16_f32(C, C, 0, 0);
      constexpr uint32_t ID_M2 = idesc_bf16_f32(C, DVT, 0, 1);
      constexpr uint32_t ID_M3 = idesc_bf16_f32(C, DVT, 0, 1);
      constexpr uint32_t ID_M4 = idesc_bf16_f32(128, DVT, 1, 1);
      const uint64_t dsb = smem_desc_sw128(smem_u32(sb_tile), G::SB_SLAB, 1024);
      // operand descriptors of stage 0 (stage s adds s * STAGE_BYTES / 16 to the
      // start-address field, which cannot carry: shared addresses are < 256 KB)
      const uint64_t dq0 = smem_desc_sw128(smem_u32(q_tile(0)), 16, 1024);          // K-major
      const uint64_t dkk0 = smem_desc_sw128(smem_u32(k_tile(0)), 16, 1024);         // K-major (scores)
      const uint64_t dkm0 = smem_desc_sw128(smem_u32(k_tile(0)), G::SLAB, 1024);    // MN-major (state update)
      const uint64_t dv0 = smem_desc_sw128(smem_u32(v_tile(0)), G::SLAB, 1024);
      const uint64_t dvd = smem_desc_sw128(smem_u32(vd_tile), G::SLAB, 1024);
      auto stage_off = [](int s) -> uint64_t { return (uint64_t)(s * (G::STAGE_BYTES >> 4)); };
      int m1_issued = 0;
      // M1 of chunk c: scores A[c%2] = qh kd^T
      auto issue_scores = [&](int c) -> bool {
        const int s = c % NS, k = c / NS, b = c & 1;
        // the transform warps saw the tile land before arriving; A[b] was last read
        // by the score step of chunk c-2, whose P tile this thread already waited for
        if (!wait_bar(sy, G::B_XFORM + s, k & 1, c)) return false;
        tc_fence_after();
        const uint64_t dq = dq0 + stage_off(s);
        const uint64_t dk = dkk0 + stage_off(s);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * G::SLAB + (kk & 3) * 32) >> 4;
          umma_bf16(tbase + G::T_A + b * C, dq + off, dk + off, ID_M1, kk > 0);
        }
        umma_commit(bars + G::B_AFULL + b);
        m1_issued = c + 1;
        return true;
      };
      int done = 0;
      if (MODE == 1) {
        // state pass: U = kd^T V per chunk; the stage is released once the state
        // update (and, normalised, the output warps' column sums) have read it
        for (int c = 0; c < nchunks; ++c) {
          const int s = c % NS, k = c / NS;
          if (!wait_bar(sy, G::B_XFORM + s, k & 1, c)) break;
          if (c > 0 && !wait_bar(sy, G::B_UEMPTY, (c - 1) & 1, c)) break;
          tc_fence_after();
          const uint64_t dvu = vd_mode ? dvd : dv0 + stage_off(s);
          const uint64_t dkd = dkm0 + stage_off(s);
#pragma unroll
          for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
              umma_bf16(tbase + G::T_U + mb * DVT, dkd + ((2 * mb * G::SLAB + kk * 2048) >> 4),
                        dvu + ((kk * 2048) >> 4), ID_M4, kk > 0);
          }
          umma_commit(bars + G::B_UFULL);
          // normalised / data-dependent decay: the state warps read the stage's key
          // sums and decay table too
          if ((NORM || GATED) && !wait_bar(sy, G::B_ZFULL + (c & 1), (c >> 1) & 1, c)) break;
          umma_commit(bars + G::B_EMPTY + s);
          done = c + 1;
        }
      }
      const int sbo = has_init ? 1 : 0;  // an initial state adds one Sb hand-over before chunk 0
      if constexpr (!GATED) {
        // A fixed order per chunk.  Three stages: M4(c), M1(c+1), M2(c), M3(c): the next
        // chunk's scores are queued before waiting for this chunk's P tile, so the score
        // step of chunk c+1 overlaps the P V product of chunk c.  Two stages (d_k = 256):
        // M4(c), M2(c), M3(c), M1(c+1): chunk c+1's tiles land only after chunk c-1's
        // stage is released.  (Measured faster than the event loop below here; the event
        // loop wins with the data-dependent decay, whose chunks wait on more barriers.)
        constexpr bool kScoresAhead = NS >= 3;
        bool ok = MODE == 1 || nchunks == 0 || issue_scores(0);
        for (int c = 0; c < nchunks && ok && MODE == 0; ++c) {
          const int s = c % NS, b = c & 1;
          const int ob = out_buf(c);
          const uint32_t oph = out_phase(c);
          const uint64_t dq = dq0 + stage_off(s);
          const uint64_t dv = dv0 + stage_off(s);
          const uint64_t dkd = dkm0 + stage_off(s);
          // M4: this chunk's state update U = kd^T V (value decay: kh^T vd)
          if (c > 0) {
            if (!wait_bar(sy, G::B_UEMPTY, (c - 1) & 1, c)) break;
            tc_fence_after();
          }
          const uint64_t dvu = vd_mode ? dvd : dv;
#pragma unroll
          for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
              umma_bf16(tbase + G::T_U + mb * DVT, dkd + ((2 * mb * G::SLAB + kk * 2048) >> 4),
                        dvu + ((kk * 2048) >> 4), ID_M4, kk > 0);
          }
          umma_commit(bars + G::B_UFULL);
          // M1 of the next chunk, ahead of M2 / M3 when three stages are in flight
          if (kScoresAhead && c + 1 < nchunks && !issue_scores(c + 1)) break;
          // M2 / M3: output accumulators
          if (!wait_bar(sy, G::B_OEMPTY + ob, oph ^ 1, c)) break;
          tc_fence_after();
          const uint32_t o_inter = tbase + G::T_O + ob * (vd_mode ? 2 : 1) * DVT;
          const uint32_t o_intra = vd_mode ? o_inter + DVT : o_inter;
          if (c > 0 || has_init) {
            if (!wait_bar(sy, G::B_SBFULL, (c - 1 + sbo) & 1, c)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * G::SLAB + (kk & 3) * 32) >> 4;
              umma_bf16(o_inter, dq + off, dsb + ((kk * 2048) >> 4), ID_M2, kk > 0);
            }
            umma_commit(bars + G::B_SBEMPTY);
          }
          if (!wait_bar(sy, G::B_PFULL + b, (c >> 1) & 1, c)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk)  // A = P from tensor memory, K = 16 per product (8 columns)
            umma_bf16_ts(o_intra, tbase + G::T_A + b * C + kk * 8, dv + ((kk * 2048) >> 4), ID_M3,
                         ((!vd_mode && (c > 0 || has_init)) || kk > 0) ? 1u : 0u);
          umma_commit(bars + G::B_OFULL + ob);
          if ((NORM || GATED) && !wait_bar(sy, G::B_ZFULL + (c & 1), (c >> 1) & 1, c)) break;  // state warps done
          umma_commit(bars + G::B_EMPTY + s);
          done = c + 1;
          if (!kScoresAhead && c + 1 < nchunks && !issue_scores(c + 1)) break;
        }
      } else {
        // Output pass: an event loop.  The thread keeps the next chunk of each product
        // (M1, M4, M2, M3) and of the stage release, and issues whichever product has
        // its operands ready (probing the barriers without blocking), M2 and M4 first:
        // they gate the state warps' serial chain (Sb -> M2 -> SBEMPTY -> next Sb, and
        // M4 -> UFULL -> S update).  Issuing in a fixed order instead leaves the tensor
        // pipe idle while one barrier is awaited and another product is ready.
        //   M1(c): stage c transformed; A[c % 2] free once the scores of chunk c - 2 are
        //          read (M3 of chunk c - 2 waited for them).
        //   M4(c): after M1(c) (stage c transformed); T_U free (UEMPTY of chunk c - 1).
        //   M2(c): after M1(c); its O buffer free (OEMPTY); Sb of chunk c (SBFULL).
        //   M3(c): after M2(c) (accumulates onto it); P(c) (PFULL).
        //   release of stage c: after all four (and, normalised or gated, ZFULL).
        int c1 = 0, c4 = 0, c2 = 0, c3 = 0, ce = 0;
        long long idle0 = clock64();
        while (MODE == 0 && ce < nchunks) {
          bool progress = false;
          if (*abort_flag) break;
          // M2(c2)
          if (c2 < c1 && mbar_test(bars + G::B_OEMPTY + out_buf(c2), out_phase(c2) ^ 1) &&
              (!(c2 > 0 || has_init) || mbar_test(bars + G::B_SBFULL, (c2 - 1 + sbo) & 1))) {
            const int c = c2, s = c % NS, ob = out_buf(c);
            if (c > 0 || has_init) {
              tc_fence_after();
              const uint32_t o_inter = tbase + G::T_O + ob * (vd_mode ? 2 : 1) * DVT;
              const uint64_t dq = dq0 + stage_off(s);
#pragma unroll
              for (int kk = 0; kk < DK / 16; ++kk) {
                const uint32_t off = ((kk >> 2) * G::SLAB + (kk & 3) * 32) >> 4;
                umma_bf16(o_inter, dq + off, dsb + ((kk * 2048) >> 4), ID_M2, kk > 0);
              }
              umma_commit(bars + G::B_SBEMPTY);
            }
            ++c2;
            progress = true;
          }
          // M4(c4)
          if (c4 < c1 && (c4 == 0 || mbar_test(bars + G::B_UEMPTY, (c4 - 1) & 1))) {
            const int c = c4, s = c % NS;
            tc_fence_after();
            const uint64_t dvu = vd_mode ? dvd : dv0 + stage_off(s);
            const uint64_t dkd = dkm0 + stage_off(s);
#pragma unroll
            for (int mb = 0; mb < G::MB; ++mb) {
#pragma unroll
              for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tbase + G::T_U + mb * DVT, dkd + ((2 * mb * G::SLAB + kk * 2048) >> 4),
                          dvu + ((kk * 2048) >> 4), ID_M4, kk > 0);
            }
            umma_commit(bars + G::B_UFULL);
            ++c4;
            progress = true;
          }
          // M3(c3)
          if (c3 < c2 && mbar_test(bars + G::B_PFULL + (c3 & 1), (c3 >> 1) & 1)) {
            const int c = c3, s = c % NS, b = c & 1, ob = out_buf(c);
            tc_fence_after();
            const uint32_t o_inter = tbase + G::T_O + ob * (vd_mode ? 2 : 1) * DVT;
            const uint32_t o_intra = vd_mode ? o_inter + DVT : o_inter;
            const uint64_t dv = dv0 + stage_off(s);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)  // A = P from tensor memory
              umma_bf16_ts(o_intra, tbase + G::T_A + b * C + kk * 8, dv + ((kk * 2048) >> 4), ID_M3,
                           ((!vd_mode && (c > 0 || has_init)) || kk > 0) ? 1u : 0u);
            umma_commit(bars + G::B_OFULL + ob);
            ++c3;
            progress = true;
          }
          // M1(c1)
          if (c1 < nchunks && c1 <= c3 + 1 && mbar_test(bars + G::B_XFORM + c1 % NS, (c1 / NS) & 1)) {
            if (!issue_scores(c1)) break;  // its wait returns at once
            c1 = m1_issued;
            progress = true;
          }
          // release of stage ce
          if (ce < c3 && ce < c4 && (!(NORM || GATED) || mbar_test(bars + G::B_ZFULL + (ce & 1), (ce >> 1) & 1))) {
            umma_commit(bars + G::B_EMPTY + ce % NS);
            ++ce;
            progress = true;
          }
          if (progress) {
            idle0 = clock64();
          } else if (clock64() - idle0 > kTimeoutCycles) {
            *abort_flag = 1;
            atomicOr(&g_tc_error, 1u);
            atomicCAS(&g_tc_where, 0u, 0x80000000u | ((uint32_t)(ce & 0x7FFFFF) << 8) | 0xFFu);
            break;
          }
        }
        if (MODE == 0) done = ce;
        if (*abort_flag) {  // products issued past the last released stage: let them finish
          const long long t = clock64();
          while (clock64() - t < 200000) {
          }
        }

      }
      // the last commits arrive asynchronously: wait for them before tensor memory is freed
      for (int c = max(0, done - NS); c < done; ++c) drain_bar(sy, G::B_EMPTY + c % NS, (c / NS) & 1);
      if (m1_issued > done) {  // a score MMA issued ahead of an aborted chunk
        const int c = m1_issued - 1;
        drain_bar(sy, G::B_AFULL + (c & 1), (c >> 1) & 1);
      }
    } else if (warp >= 2) {
      // ========================================================== transform
      // 64 threads; thread tt owns the 16-byte vectors tt + 64 m of a tile.  A
      // vector v sits in row (v mod 8C) / 8 of its [C x 64] slab.
      const int tt = tid - 64;
      constexpr bool elu = ELU;
      // vectors per thread of a q or k tile: 8 per 64-column slab; a d_k of 64 in the
      // d_k = 128 layout transforms slab 0 only (slab 1 holds TMA zero fill, which
      // must stay zero: phi(0) = 1 for elu + 1)
      const int NV = 8 * (a.dk / 64);
      constexpr int NVV = G::V_BYTES / 16 / 64;   // ... of a v tile
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % NS, k = c / NS;
        if (!wait_bar(sy, G::B_FULL + s, k & 1, c)) break;
        const int Cp = chunk_len(c);
        if (vd_mode && c > 0 && !wait_bar(sy, G::B_UFULL, (c - 1) & 1, c)) break;  // M4(c-1) read vd
        static_assert(G::SLAB / 16 == 8 * 64, "row mapping assumes C = 64");
        // Data-dependent decay: prefix sums b_i = sum_{t<=i} log alpha_t over the
        // chunk (tokens past its end count as alpha = 1).  Each warp computes all
        // 64 (lane l holds b_l and b_{l+32}); the first warp publishes them with
        // b_last = b_{C'-1} in the stage's table.
        float blo = 0.f, bhi = 0.f, blast = 0.f;
        if (GATED) {
          const int ln = tt & 31;
          if (REV) {  // position p: the decay of the token after it (reversed order), none after the last
            const int64_t after0 = (int64_t)bidx * a.T + rend - (int64_t)c * C;  // token after position 0
            blo = (ln < Cp && (c > 0 || ln > 0)) ? a.g[(after0 - ln) * a.H + h] : 0.f;
            bhi = ln + 32 < Cp ? a.g[(after0 - ln - 32) * a.H + h] : 0.f;
          } else {
            const int64_t row0 = (int64_t)bidx * a.T + start + (int64_t)c * C;
            blo = ln < Cp ? a.g[(row0 + ln) * a.H + h] : 0.f;
            bhi = ln + 32 < Cp ? a.g[(row0 + ln + 32) * a.H + h] : 0.f;
          }
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, blo, o);
            const float y1 = __shfl_up_sync(0xffffffffu, bhi, o);
            if (ln >= o) {
              blo += y0;
              bhi += y1;
            }
          }
          bhi += __shfl_sync(0xffffffffu, blo, 31);
          blast = __shfl_sync(0xffffffffu, Cp <= 32 ? blo : bhi, (Cp - 1) & 31);
          if (tt < 32) {
            float *dt = dtab + s * G::DT_STRIDE;
            dt[ln] = blo;
            dt[ln + 32] = bhi;
            if (ln == 0) dt[C] = blast;
          }
        }
        // row weights of this thread's vectors: gamma^(C'-1-j) (data-dependent:
        // exp(b_last - b_j)), zero past the chunk end
        auto decay_weights = [&](float (&wv)[8]) {
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int j = (tt >> 3) + 8 * m;
            if (GATED) {  // the table is indexed by position (reversed order in reverse time)
              const int jp = lrow(j);
              const float b0 = __shfl_sync(0xffffffffu, blo, jp & 31);
              const float b1 = __shfl_sync(0xffffffffu, bhi, jp & 31);
              wv[m] = jp < Cp ? exp_fast(blast - (jp < 32 ? b0 : b1)) : 0.f;
            } else {
              const int jl = lrow(j);
              wv[m] = jl < Cp ? pw[Cp - 1 - jl] : 0.f;
            }
          }
        };
        float wv[8], wsum[8];
        // keys: phi, and the decay unless in value-decay mode (which keeps phi(k)
        // as is); the queries are the output warps' part.  Normalised, the pass
        // also leaves the chunk's weighted key column sums (gamma^(C'-1-j) on row
        // j, zero past the chunk end) in ksum[s], one row per warp.
        float *ks = ksum + (s * 2 + (tt >> 5)) * DK;
        const bool store_k = elu || (!vd_mode && (g != 1.f || Cp != C));
        if (vd_mode) {
#pragma unroll
          for (int m = 0; m < 8; ++m) wv[m] = 1.f;
          decay_weights(wsum);
        } else {
          decay_weights(wv);
#pragma unroll
          for (int m = 0; m < 8; ++m) wsum[m] = wv[m];
        }
        if (store_k)
          xform_tile<ELU, true, NORM>(k_tile(s), k_tile(s), tt, NV, wv, wsum, ks);
        else if (NORM)
          xform_tile<false, false, true>(k_tile(s), k_tile(s), tt, NV, wv, wsum, ks);
        // value-decay mode: decayed values vd for the state update
        if (vd_mode) {
          decay_weights(wv);
          xform_tile<false, true, false>(v_tile(s), vd_tile, tt, NVV, wv, wv, ks);
        }
        fence_proxy_async_smem();
        mbar_arrive(bars + G::B_XFORM + s);
      }
    }
  } else if (warp < 8) {
    // ================================================================ state
    reg_alloc<232>();
    const int sp = warp & 3;
    float S[G::RPT];
    if (has_init) {  // start state of this segment, from the scan (S^T rows)
      const float *W = a.ws_s + ws_slot * DK * DVT;
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
        const float4 *src = reinterpret_cast<const float4 *>(W + (mb * 128 + sp * 32 + lane) * DVT);
#pragma unroll
        for (int q = 0; q < DVT / 4; ++q) {
          const float4 x = src[q];
          S[mb * DVT + 4 * q] = x.x;
          S[mb * DVT + 4 * q + 1] = x.y;
          S[mb * DVT + 4 * q + 2] = x.z;
          S[mb * DVT + 4 * q + 3] = x.w;
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < G::RPT; ++u) S[u] = 0.f;
    }
    // normaliser key sums z[kr] for the rows this thread holds
    float zr[G::MB];
#pragma unroll
    for (int mb = 0; mb < G::MB; ++mb)
      zr[mb] = (NORM && has_init) ? a.ws_z[ws_slot * DK + mb * 128 + sp * 32 + lane] : 0.f;
    // z <- gdec z + (chunk c's weighted key column sums, from the transform
    // warps), published in z buffer (c & 1) for the output warps; gdec is the
    // chunk's whole decay (gamma^C' or exp(b_last))
    auto key_sums = [&](int c, float gdec) -> bool {
      const int s = c % NS;
      if (!wait_bar_warp(sy, G::B_XFORM + s, (c / NS) & 1, c)) return false;
      const float *ks = ksum + s * 2 * DK;
      float *zb = z + (c & 1) * DK;
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
        const int kr = mb * 128 + sp * 32 + lane;
        zr[mb] = kr < a.dk ? fmaf(gdec, zr[mb], ks[kr] + ks[DK + kr]) : 0.f;
        zb[kr] = zr[mb];
      }
      return true;
    };
    float seg_log = 0.f;  // data-dependent decay: log of this segment's whole decay (state pass)
    // bf16 operand Sb = sc * S for the next chunk's inter-chunk product
    auto write_sb = [&](float sc) {
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
        const int kr = mb * 128 + sp * 32 + lane;  // d_k index held by this thread
#pragma unroll
        for (int grp = 0; grp < DVT / 32; ++grp) {
          uint8_t *row = sb_tile + ((grp * 32) >> 6) * G::SB_SLAB + kr * 128;
          const int ch0 = ((grp * 32) & 63) >> 3;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float *x = &S[mb * DVT + grp * 32 + 8 * q];
            const uint4 v = make_uint4(pack2(sc * x[0], sc * x[1]), pack2(sc * x[2], sc * x[3]),
                                       pack2(sc * x[4], sc * x[5]), pack2(sc * x[6], sc * x[7]));
            *reinterpret_cast<uint4 *>(row + (((ch0 + q) ^ (kr & 7)) << 4)) = v;
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bars + G::B_SBFULL);
    };
    const int sbo = has_init ? 1 : 0;
    if (has_init && nchunks > 0) write_sb(vd_mode ? 1.f : pw[chunk_len(0)]);
    for (int c = 0; c < nchunks; ++c) {
      const int Cp = chunk_len(c);
      if (!wait_bar_warp(sy, G::B_UFULL, c & 1, c)) break;
      tc_fence_after();
      float gdec = pw[Cp];
      if (GATED) {  // the chunk's decay from the transform warps' table
        if (!wait_bar_warp(sy, G::B_XFORM + c % NS, (c / NS) & 1, c)) break;
        const float bl = dtab[(c % NS) * G::DT_STRIDE + C];
        gdec = exp_fast(bl);
        seg_log += bl;
      }
      // two 32-column loads in flight per wait
#pragma unroll
      for (int g2 = 0; g2 < G::RPT / 64; ++g2) {
        uint32_t r0[32], r1[32];
        const uint32_t col = G::T_U + g2 * 64;  // state values [64 g2, 64 g2 + 64) of this thread
        tmem_ld_32x32b_x32(tbase + ((uint32_t)(sp * 32) << 16) + col, r0);
        tmem_ld_32x32b_x32(tbase + ((uint32_t)(sp * 32) << 16) + col + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          S[g2 * 64 + e] = fmaf(gdec, S[g2 * 64 + e], __uint_as_float(r0[e]));
          S[g2 * 64 + 32 + e] = fmaf(gdec, S[g2 * 64 + 32 + e], __uint_as_float(r1[e]));
        }
      }
      tc_fence_before();
      mbar_arrive(bars + G::B_UEMPTY);
      if (NORM && !key_sums(c, gdec)) break;
      // this warpgroup is done with the stage's key sums and decay table
      if (NORM || GATED) mbar_arrive(bars + G::B_ZFULL + (c & 1));
      if (MODE == 1 || c == nchunks - 1) continue;
      // the previous Sb has been read once M2 of chunk c is done
      if (c - 1 + sbo >= 0 && !wait_bar_warp(sy, G::B_SBEMPTY, (c - 1 + sbo) & 1, c)) break;
      write_sb(vd_mode ? 1.f : pw[chunk_len(c + 1)]);
    }
    // S after the last chunk: the segment's end state (state pass) or the final
    // state of the sequence (zero for an empty sequence)
    float *F = nullptr;
    int64_t ld = a.dv;
    if (MODE == 1) {
      F = a.ws_s + ws_slot * DK * DVT;
      ld = DVT;
      if (NORM) {
#pragma unroll
        for (int mb = 0; mb < G::MB; ++mb) a.ws_z[ws_slot * DK + mb * 128 + sp * 32 + lane] = zr[mb];
      }
      if (GATED && sp == 0 && lane == 0) a.ws_g[ws_slot] = seg_log;
    } else if (a.final_state && last_seg) {
      F = a.final_state + ((int64_t)n * a.H + h) * (int64_t)a.dk * a.dv + vt * DVT;
    }
    if (MODE == 0 && NORM && a.final_z && last_seg && vt == 0) {  // z after the last token
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
        const int kr = mb * 128 + sp * 32 + lane;
        if (kr < a.dk) a.final_z[((int64_t)n * a.H + h) * a.dk + kr] = zr[mb];
      }
    }
    if (F) {  // workspace slots hold all DK x DVT values; the final state only d_k rows, d_v columns
      const int rows = MODE == 1 ? DK : a.dk;
      const int cols = MODE == 1 ? DVT : min(DVT, a.dv - vt * DVT);
#pragma unroll
      for (int mb = 0; mb < G::MB; ++mb) {
        const int kr = mb * 128 + sp * 32 + lane;
        float4 *dst = reinterpret_cast<float4 *>(F + (int64_t)kr * ld);
        if (kr < rows) {
#pragma unroll
          for (int q = 0; q < DVT / 4; ++q)
            if (4 * q < cols)
              dst[q] = make_float4(S[mb * DVT + 4 * q], S[mb * DVT + 4 * q + 1], S[mb * DVT + 4 * q + 2],
                                   S[mb * DVT + 4 * q + 3]);
        }
      }
    }
  } else {
    // ================================================================ output
    // The kernel launches with 168 registers per thread (384 threads); the
    // warpgroups re-split them as 104 (producer, MMA, transform), 232 (state)
    // and 168 (output), 504 x 128 in total.  setmaxnreg.inc may only raise and
    // .dec only lower a warp's count; the output warpgroup keeps the launch count.
    const int sp = warp & 3;
    const int i = sp * 16 + (lane & 15);  // chunk row held by this thread
    const int hf = lane >> 4;             // which half of the columns
    uint8_t *obase = reinterpret_cast<uint8_t *>(a.out) +
                     2 * ((int64_t)bidx * a.o_sb + (int64_t)h * a.o_sh + vt * DVT);

    // zq = z_p . qh_i over this thread's row and column half, z_p = z before chunk c
    // (z buffer (c - 1) & 1; for c = 0 buffer 1 holds the initial z).  The q tile
    // is final: the score MMA of chunk c has read it.
    auto z_dot_q = [&](int c, bool &ok) -> float {
      ok = false;
      if (c > 0 && !wait_bar_warp(sy, G::B_ZFULL + ((c - 1) & 1), ((c - 1) >> 1) & 1, c)) return 0.f;
      const float *zp = z + ((c - 1) & 1) * DK;
      const uint8_t *qt = q_tile(c % NS);
      float zq = 0.f;
      // columns in logical order (8-column block p sits in 16-byte chunk p ^ (i & 7)
      // of the row): every lane of a half-warp reads the same z values
#pragma unroll
      for (int kb = hf * (G::KB / 2); kb < (hf + 1) * (G::KB / 2); ++kb) {
        const uint8_t *row = qt + kb * G::SLAB + i * 128;
        uint4 qv[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) qv[p] = *reinterpret_cast<const uint4 *>(row + ((p ^ (i & 7)) << 4));
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float *zc = zp + kb * 64 + p * 8;
          const float4 z0 = *reinterpret_cast<const float4 *>(zc);
          const float4 z1 = *reinterpret_cast<const float4 *>(zc + 4);
          float f[8];
          unpack8(qv[p], f);
          zq = fmaf(z0.x, f[0], zq); zq = fmaf(z0.y, f[1], zq); zq = fmaf(z0.z, f[2], zq);
          zq = fmaf(z0.w, f[3], zq); zq = fmaf(z1.x, f[4], zq); zq = fmaf(z1.y, f[5], zq);
          zq = fmaf(z1.z, f[6], zq); zq = fmaf(z1.w, f[7], zq);
        }
      }
      zq += __shfl_xor_sync(0xffffffffu, zq, 16);
      ok = true;
      return zq;
    };

    // scores of chunk c -> P tile; returns this row's output factor and, in
    // value-decay mode, the inter-chunk factor gi (gamma^(i+1) or exp(b_i))
    auto scores = [&](int c, bool &ok, float &gi) -> float {
      const int b = c & 1;
      const int Cp = chunk_len(c);
      ok = false;
      if (!wait_bar_warp(sy, G::B_AFULL + b, (c >> 1) & 1, c)) return 0.f;
      tc_fence_after();
      if (NG && lrow(i) < Cp) {  // warm L2 with this row's gate for the epilogue of chunk c (one step later)
        const uint8_t *gp = reinterpret_cast<const uint8_t *>(a.ng_gate) +
                            2 * ((int64_t)bidx * a.ng_sb + (int64_t)h * a.ng_sh + (tok0(c) + i) * a.ng_st +
                                 hf * (DVT / 2));
#pragma unroll
        for (int l = 0; l < DVT; l += 64) asm volatile("prefetch.global.L2 [%0];" ::"l"(gp + l));
      }
      const float *dt = dtab + (c % NS) * G::DT_STRIDE;
      float bi = 0.f;
      if (GATED) {  // the stage's decay table (published before the score MMA's inputs)
        if (!wait_bar_warp(sy, G::B_XFORM + c % NS, (c / NS) & 1, c)) return 0.f;
        bi = dt[lrow(i)];
        gi = exp_fast(bi);
      } else {
        gi = pw[lrow(i) + 1];
      }
      float zq = 0.f;
      if (NORM) {
        zq = z_dot_q(c, ok);
        if (!ok) return 0.f;
        ok = false;
      }
      uint32_t r[32];
      tmem_ld_16x32bx2_x32<32>(tbase + ((uint32_t)(sp * 32) << 16) + G::T_A + b * C, r);
      tmem_wait_ld();
      float f[32];
      const int il = lrow(i);  // row of the (reversed) sequence
      const bool row_ok = il < Cp;
      if (REV) {  // causal in the reversed order: j' <= i', i.e. j >= i
        if (!vd_mode) {
#pragma unroll
          for (int e = 0; e < 32; ++e) f[e] = (hf * 32 + e >= i && row_ok) ? __uint_as_float(r[e]) : 0.f;
        } else if (GATED) {  // P_ij = A_ij exp(b''_i' - b''_j') over reversed positions
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = hf * 32 + e;
            f[e] = (j >= i && row_ok) ? __uint_as_float(r[e]) * exp_fast(bi - dt[lrow(j)]) : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = hf * 32 + e;
            f[e] = (j >= i && row_ok) ? __uint_as_float(r[e]) * pw[j - i] : 0.f;
          }
        }
      } else if (!vd_mode) {
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = (hf * 32 + e <= i && row_ok) ? __uint_as_float(r[e]) : 0.f;
      } else if (GATED) {  // P_ij = A_ij exp(b_i - b_j)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = hf * 32 + e;
          f[e] = (j <= i && row_ok) ? __uint_as_float(r[e]) * exp_fast(bi - dt[j]) : 0.f;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = hf * 32 + e;
          f[e] = (j <= i && row_ok) ? __uint_as_float(r[e]) * pw[i - j] : 0.f;
        }
      }
      {  // P in tensor memory, in place: row i's columns [32 hf, 32 hf + 32) as bf16 pairs in score
         // columns [16 hf, 16 hf + 16) (the M = 64 layout: row 16 w + l at lane 32 w + l); this
         // warp has read its lanes of the fp32 tile already
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack2(f[2 * e], f[2 * e + 1]);
        tmem_st_16x32bx2_x16<16>(tbase + ((uint32_t)(sp * 32) << 16) + G::T_A + b * C, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bars + G::B_PFULL + b);  // also tells the MMA issuer that A[b] has been read
      ok = true;
      float rowsum = 0.f;
      if (NORM) {  // warp-wide: every lane takes part, including rows past the chunk end
#pragma unroll
        for (int e = 0; e < 32; ++e) rowsum += f[e];
        rowsum += __shfl_xor_sync(0xffffffffu, rowsum, 16);
      }
      if (!row_ok) return 0.f;
      if (!NORM) return vd_mode ? 1.f : 1.f / pw[Cp - 1 - il];
      return 1.f / fmaf(vd_mode ? gi : pw[Cp], zq, rowsum);
    };

    // epilogue of chunk c
    auto epilogue = [&](int c, float fac, float gi) -> bool {
      const int Cp = chunk_len(c);
      const int ob = out_buf(c);
      const uint32_t oph = out_phase(c);
      const int64_t otok = tok0(c) + i;  // natural token of this row (in reverse time, may precede the sequence)
      if (!wait_bar_warp(sy, G::B_OFULL + ob, oph, c)) return false;
      tc_fence_after();
      const uint32_t lane_base = tbase + ((uint32_t)(sp * 32) << 16);
      // this thread's 32 output values of a pass (columns hf DVT/2 + 32 pass ...)
      auto load_o = [&](int pass, float (&o)[32]) {
        uint32_t ra[32], re[32];
        if (vd_mode) {  // o = gamma^(i+1) O_inter + O_intra; no inter term without a prior state
          const bool inter = c > 0 || has_init;
          const uint32_t pair = lane_base + G::T_O + ob * 2 * DVT + pass * 32;
          tmem_ld_16x32bx2_x32<DVT / 2>(pair + DVT, ra);
          if (inter) tmem_ld_16x32bx2_x32<DVT / 2>(pair, re);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            o[e] = fmaf(gi, inter ? __uint_as_float(re[e]) : 0.f, __uint_as_float(ra[e])) * fac;
        } else {
          tmem_ld_16x32bx2_x32<DVT / 2>(lane_base + G::T_O + ob * DVT + pass * 32, ra);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(ra[e]) * fac;
        }
      };
      float rstd = 1.f;
      if (NG) {  // output norm: the row's mean square over d_v (this thread and its other half, lane ^ 16)
        float ss = 0.f;
#pragma unroll 1
        for (int pass = 0; pass < DVT / 64; ++pass) {
          float o[32];
          load_o(pass, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) ss = fmaf(o[e], o[e], ss);
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 16);
        rstd = rsqrtf(ss / (float)DVT + a.ng_eps);
      }
      float edot = 0.f;  // backward epilogue: this thread's part of phi(x) . o
      auto do_pass = [&](int pass) {
        float o[32];
        load_o(pass, o);
        if (pass == DVT / 64 - 1) {
          tc_fence_before();
          mbar_arrive(bars + G::B_OEMPTY + ob);
        }
        const int col = hf * (DVT / 2) + pass * 32;
        if (lrow(i) < Cp && vt * DVT + col < a.dv) {
          if (!NG && a.ex) {  // the row of x at this token: the dot takes o before phi' scales it
            const uint4 *xs = reinterpret_cast<const uint4 *>(
                reinterpret_cast<const uint8_t *>(a.ex) +
                2 * ((int64_t)bidx * a.ex_sb + otok * a.ex_st + (int64_t)h * a.ex_sh + vt * DVT + col));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float xf[8];
              unpack8(xs[q], xf);
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const float xv = xf[u];
                edot = fmaf(a.ephi ? phi_fast(xv) : xv, o[8 * q + u], edot);
                if (a.edphi) o[8 * q + u] *= xv > 0.f ? 1.f : exp_fast(xv);
              }
            }
          }
          if (NG) {  // y = o rstd w swish(gate)
            const uint4 *gsrc = reinterpret_cast<const uint4 *>(
                reinterpret_cast<const uint8_t *>(a.ng_gate) +
                2 * ((int64_t)bidx * a.ng_sb + (int64_t)h * a.ng_sh + otok * a.ng_st + col));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float gv[8];
              unpack8(gsrc[q], gv);
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int e = 8 * q + u;
                o[e] = o[e] * rstd * ngw[col + e] * swish_fast(gv[u]);
              }
            }
          }
          uint4 *dst = reinterpret_cast<uint4 *>(obase + 2 * (otok * a.o_st + col));
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack2(o[8 * q], o[8 * q + 1]), pack2(o[8 * q + 2], o[8 * q + 3]),
                                pack2(o[8 * q + 4], o[8 * q + 5]), pack2(o[8 * q + 6], o[8 * q + 7]));
        }
      };
#pragma unroll 1
      for (int pass = 0; pass < DVT / 64; ++pass) do_pass(pass);
      if (!NG && a.edg) {  // the row's two halves, then one thread adds the row's term
        edot += __shfl_xor_sync(0xffffffffu, edot, 16);
        if (hf == 0 && lrow(i) < Cp) atomicAdd(a.edg + ((int64_t)bidx * a.T + otok) * a.H + h, a.esign * edot);
      }
      // the row's denominator: fac is 1 / den, or in decayed-key mode 1 / (den gamma^(C'-1-i))
      if (NORM && a.den_out && vt == 0 && hf == 0 && lrow(i) < Cp)
        a.den_out[((int64_t)bidx * a.T + otok) * a.H + h] =
            vd_mode ? 1.f / fac : 1.f / (fac * pw[Cp - 1 - lrow(i)]);
      return true;
    };

    // elu + 1 on chunk c's query tile: this thread's row and column half, in place
    // (chunks in the same conflict-free order as above)
    auto q_xform = [&](int c) -> bool {
      const int s = c % NS;
      if (!wait_bar_warp(sy, G::B_FULL + s, (c / NS) & 1, c)) return false;
#pragma unroll 1
      for (int kb = hf * (G::KB / 2); kb < (hf + 1) * (G::KB / 2) && kb < a.dk / 64; ++kb) {
        uint8_t *row = q_tile(s) + kb * G::SLAB + i * 128;
        uint4 x[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) x[p] = *reinterpret_cast<const uint4 *>(row + ((p ^ (i & 7)) << 4));
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          float f[8];
          unpack8(x[p], f);
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] = phi_fast(f[u]);
          *reinterpret_cast<uint4 *>(row + ((p ^ (i & 7)) << 4)) = pack8(f);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bars + G::B_XFORM + s);
      return true;
    };

    // scores run one chunk ahead of the epilogue: step t does scores(t), epilogue(t-1)
    // and, with elu + 1, the query transform of chunk t + NS - 1 (the first NS - 1
    // before the loop), so that the score MMA never waits for it
    constexpr int QLA = NS - 1;
    bool qok = true;
    if (kQByOutput)
      for (int c = 0; c < QLA && c < nchunks && qok; ++c) qok = q_xform(c);
    float fac_even = 0.f, fac_odd = 0.f, gi_even = 0.f, gi_odd = 0.f;
    for (int t = 0; t <= nchunks && MODE == 0 && qok; ++t) {
      if (t < nchunks) {
        bool ok = true;
        float gi = 0.f;
        const float f = scores(t, ok, gi);
        if (!ok) break;
        if (t & 1) {
          fac_odd = f;
          gi_odd = gi;
        } else {
          fac_even = f;
          gi_even = gi;
        }
      }
      if (t >= 1 && !epilogue(t - 1, ((t - 1) & 1) ? fac_odd : fac_even, ((t - 1) & 1) ? gi_odd : gi_even)) break;
      if (kQByOutput && t + QLA < nchunks && !q_xform(t + QLA)) break;
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    tmem_dealloc(tbase, G::T_COLS);
    tmem_relinquish();
  }
}

// ---------------------------------------------------------------- host side

// Segmentation plan for the tensor-core path: when a dense batch has too few
// (sequence, head, value-slice) units to fill the GPU, every sequence is split
// into G segments of segC chunks so that units * G CTAs run in one wave.  The
// plan depends only on the problem shape (not on the device), so the workspace
// size a caller queries matches what the launch uses.
constexpr int kPlanSMs = 148;         // B200 streaming multiprocessors
constexpr int kMinSegmentChunks = 16;  // below this the two extra passes do not pay

struct SegPlan {
  int G = 1, segC = 0;
  int64_t units = 0;
};

// Value-slice width of the tensor-core kernel for a key head dim: the state
// warpgroup holds d_k x DVT fp32 values, 128 per thread.  d_k = 64 runs in the
// d_k = 128 layout (key and query columns 64 .. 127 are TMA zero fill).
constexpr int tc_dvt(int dk) { return dk == 256 ? 64 : 128; }
constexpr int tc_dk(int dk) { return dk == 256 ? 256 : 128; }
// Value slices of a d_v: a d_v of 64 in a 128-wide slice counts as one.
inline int tc_nvt(int dk, int dv) { return (dv + tc_dvt(dk) - 1) / tc_dvt(dk); }

SegPlan seg_plan(int64_t n_seqs, int64_t T, int64_t H, int nvt, bool varlen, int chunk) {
  SegPlan p;
  p.units = n_seqs * H * nvt;
  if (varlen || p.units <= 0 || T <= 0) return p;
  const int64_t nch = (T + chunk - 1) / chunk;
  int64_t G = kPlanSMs / p.units;
  if (nch / kMinSegmentChunks < G) G = nch / kMinSegmentChunks;
  if (G < 2) return p;
  const int64_t segC = (nch + G - 1) / G;
  p.G = (int)((nch + segC - 1) / segC);
  p.segC = (int)segC;
  if (p.G < 2) p.G = 1;
  return p;
}

// Workspace of a segmented launch: segment states S^T [units][G-1][dk][dvt],
// normaliser sums [units][G-1][dk], segment log decays [units][G-1].
size_t seg_ws_bytes(const SegPlan &p, int dk, int dvt) {
  if (p.G < 2) return 0;
  return (size_t)p.units * (p.G - 1) * ((size_t)dk * dvt + dk + 1) * sizeof(float);
}

// Packed batches run their sequences longest first: CTAs start in index order,
// so the long sequences no longer finish last on a few SMs (a schedule
// simulation of a 64-sequence batch of lengths U[128, 2048] gives an 11%
// shorter makespan).  The order lives in the workspace, after any segment
// states; above kOrderMaxSeqs sequences the natural order is kept.
constexpr int64_t kOrderMaxSeqs = 4096;

size_t order_bytes(int64_t n_seqs, bool varlen) {
  if (!varlen || n_seqs < 2 || n_seqs > kOrderMaxSeqs) return 0;
  return ((size_t)n_seqs * sizeof(int32_t) + 255) / 256 * 256;
}

// order[rank] = the sequence of that rank: longer first, ties by index.  One
// thread per sequence counts the sequences that rank before it.
__global__ void seq_order_kernel(const int32_t *cu, int n, int32_t *order) {
  extern __shared__ int32_t lens[];
  for (int m = threadIdx.x; m < n; m += blockDim.x) lens[m] = cu[m + 1] - cu[m];
  __syncthreads();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int li = lens[i];
  int r = 0;
  for (int m = 0; m < n; ++m) r += (lens[m] > li) || (lens[m] == li && m < i);
  order[r] = i;
}

// Segment start states from segment end states, in place: slot g-1 of a unit
// ends up holding W_g = D_{g-1} W_{g-1} + E_{g-1} (W_0 = 0), where D is the
// decay over a full segment: gamma^L (L tokens), or exp of the segment's summed
// log decay (ws_g) with a data-dependent decay; the same recurrence runs on the
// normaliser sums.
__global__ void seg_scan_kernel(float *ws_s, float *ws_z, const float *ws_g, const float *gamma, int G,
                                int64_t seg_tokens, int H, int nvt, int elems_s, int elems_z) {
  const int64_t unit = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= elems_s + elems_z) return;
  const int h = (int)((unit / nvt) % H);
  const float gL = ws_g ? 0.f : powf(gamma[h], (float)seg_tokens);
  float *base;
  int64_t stride;
  if (e < elems_s) {
    base = ws_s + unit * (int64_t)(G - 1) * elems_s + e;
    stride = elems_s;
  } else {
    if (!ws_z) return;
    base = ws_z + unit * (int64_t)(G - 1) * elems_z + (e - elems_s);
    stride = elems_z;
  }
  float w = 0.f;
  for (int g = 1; g < G; ++g) {
    float *slot = base + (int64_t)(g - 1) * stride;
    const float d = ws_g ? expf(ws_g[unit * (G - 1) + (g - 1)]) : gL;
    w = fmaf(d, w, *slot);
    *slot = w;
  }
}

template <int DK, int DVT, int C, int NS, bool NORM, bool ELU, bool GATED, bool REV, bool NG = false>
cudaError_t launch_cfg(const ChunkArgs &a, void *workspace, cudaStream_t stream, const char **why) {
  using G = Cfg<DK, DVT, C, NS>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.B, a.T, a.H, a.dk, C) || !make_map(&mk, a.k, a.B, a.T, a.H, a.dk, C) ||
      !make_map(&mv, a.v, a.B, a.T, a.H, a.dv, C)) {
    if (why) *why = "cuTensorMapEncodeTiled rejected a tensor";
    return cudaErrorInvalidValue;
  }
  TcArgs t;
  t.out = a.out;
  t.o_sb = a.o_sb;
  t.o_st = a.o_st;
  t.o_sh = a.o_sh;
  t.gamma = a.gamma;
  t.cu_seqlens = a.cu_seqlens;
  t.final_state = a.final_state;
  t.final_z = a.final_z;
  t.g = a.g;
  t.T = a.T;
  t.H = a.H;
  t.dk = a.dk;
  t.dv = a.dv;
  t.phi = a.phi;
  t.normalize = a.normalize;
  const int nvt = (a.dv + DVT - 1) / DVT;
  const SegPlan plan = a.noseg ? SegPlan{1, 0, 0} : seg_plan(a.n_seqs, a.T, a.H, nvt, a.cu_seqlens != nullptr, C);
  const int64_t units = a.n_seqs * a.H * nvt;
  if (units == 0) return cudaSuccess;
  if (units * plan.G > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  t.G = plan.G;
  t.segC = plan.segC;
  t.ws_s = nullptr;
  t.ws_z = nullptr;
  t.ws_g = nullptr;
  t.order = nullptr;
  t.ng_w = a.ng_w;
  t.ng_gate = a.ng_gate.data;
  t.ng_sb = a.ng_gate.sb;
  t.ng_st = a.ng_gate.st;
  t.ng_sh = a.ng_gate.sh;
  t.ng_eps = a.ng_eps;
  t.ex = a.ex.data;
  t.ex_sb = a.ex.sb;
  t.ex_st = a.ex.st;
  t.ex_sh = a.ex.sh;
  t.edg = a.edg;
  t.esign = a.esign;
  t.ephi = a.ephi;
  t.edphi = a.edphi;
  t.den_out = a.den_out;
  const size_t ob = a.noseg ? 0 : order_bytes(a.n_seqs, a.cu_seqlens != nullptr);
  if (ob > 0 && workspace) {
    int32_t *order = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + seg_ws_bytes(plan, DK, DVT));
    const int nn = (int)a.n_seqs;
    seq_order_kernel<<<(nn + 255) / 256, 256, nn * sizeof(int32_t), stream>>>(a.cu_seqlens, nn, order);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    t.order = order;
  }
  auto kern = chunk_tc_kernel<DK, DVT, C, NS, NORM, ELU, 0, GATED, REV, NG>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  if (plan.G > 1) {
    if (!workspace) {
      if (why) *why = "segmented launch without workspace";
      return cudaErrorInvalidValue;
    }
    t.ws_s = static_cast<float *>(workspace);
    t.ws_z = NORM ? t.ws_s + units * (plan.G - 1) * DK * DVT : nullptr;
    t.ws_g = GATED ? t.ws_s + units * (plan.G - 1) * (DK * DVT + DK) : nullptr;
    // pass 1: end state of every segment but the last, from a zero start
    auto kst = chunk_tc_kernel<DK, DVT, C, NS, NORM, ELU, 1, GATED, REV>;
    err = cudaFuncSetAttribute(kst, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    t.Gp = plan.G - 1;
    kst<<<(unsigned)(units * t.Gp), kThreads, G::SMEM_BYTES, stream>>>(mq, mk, mv, t);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    // scan: start states of segments 1 .. G-1
    const int elems_s = DK * DVT, elems_z = NORM ? DK : 0;
    dim3 sgrid((unsigned)((elems_s + elems_z + 255) / 256), (unsigned)units);
    seg_scan_kernel<<<sgrid, 256, 0, stream>>>(t.ws_s, t.ws_z, t.ws_g, a.gamma, plan.G, (int64_t)plan.segC * C,
                                               a.H, nvt, elems_s, elems_z);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  // output pass: every segment, seeded with its start state
  t.Gp = plan.G;
  kern<<<(unsigned)(units * plan.G), kThreads, G::SMEM_BYTES, stream>>>(mq, mk, mv, t);
  return cudaGetLastError();
}

}  // namespace

cudaError_t tc_device_error(unsigned int *flags, unsigned int *where, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_tc_error, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(where, g_tc_where, sizeof(unsigned int));
  if (e == cudaSuccess && reset) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_tc_where, &zero, sizeof(zero));
  }
  return e;
}

// The output norm fuses into the epilogue when one CTA holds whole rows of d_v.
bool tc_can_fuse_norm_gate(const ChunkArgs &a) {
  return (a.dk == 64 || a.dk == 128) && a.dv == tc_dvt(a.dk) && !a.g && !a.rev;
}

// Head dims the tensor-core kernel takes: d_k in {64, 128} with d_v = 64 or a
// multiple of 128, and d_k = 256 with d_v a multiple of 64.
bool tc_shape(int dk, int dv) {
  if (dk == 64 || dk == 128) return dv == 64 || (dv > 0 && dv % 128 == 0);
  if (dk == 256) return dv > 0 && dv % 64 == 0;
  return false;
}

bool tc_supported(const ChunkArgs &a) {
  if (a.dtype != LA_BF16 || a.chunk != 64) return false;
  if (!tc_shape(a.dk, a.dv)) return false;
  if (a.T > 0x7fffffffLL || a.H > 0xffff) return false;
  return encode_fn() != nullptr;
}

size_t tc_workspace_bytes(int64_t B, int64_t T, int64_t H, int dk, int dv, int64_t n_seqs, bool varlen, int chunk) {
  (void)B;
  if (chunk != 64 || !tc_shape(dk, dv)) return 0;  // not a tensor-core shape
  return seg_ws_bytes(seg_plan(n_seqs, T, H, tc_nvt(dk, dv), varlen, chunk), tc_dk(dk), tc_dvt(dk)) +
         order_bytes(n_seqs, varlen);
}

template <int DK, int DVT, int NS, bool GATED>
cudaError_t launch_shape_gated(const ChunkArgs &a, void *workspace, cudaStream_t stream, const char **why) {
  // one instantiation per (normaliser, feature map, decay kind): each carries only its own code path
  if (!GATED && DVT == 128 && a.ng_w) {  // output norm and gate fused into the epilogue
    if (a.dv != DVT) return cudaErrorInvalidValue;
    if (a.normalize)
      return a.phi ? launch_cfg<DK, DVT, 64, NS, true, true, false, false, true>(a, workspace, stream, why)
                   : launch_cfg<DK, DVT, 64, NS, true, false, false, false, true>(a, workspace, stream, why);
    return a.phi ? launch_cfg<DK, DVT, 64, NS, false, true, false, false, true>(a, workspace, stream, why)
                 : launch_cfg<DK, DVT, 64, NS, false, false, false, false, true>(a, workspace, stream, why);
  }
  if (a.normalize) {
    return a.phi ? launch_cfg<DK, DVT, 64, NS, true, true, GATED, false>(a, workspace, stream, why)
                 : launch_cfg<DK, DVT, 64, NS, true, false, GATED, false>(a, workspace, stream, why);
  }
  return a.phi ? launch_cfg<DK, DVT, 64, NS, false, true, GATED, false>(a, workspace, stream, why)
               : launch_cfg<DK, DVT, 64, NS, false, false, GATED, false>(a, workspace, stream, why);
}

template <int DK, int DVT, int NS>
cudaError_t launch_shape(const ChunkArgs &a, void *workspace, cudaStream_t stream, const char **why) {
  if (a.rev) {  // reverse time (the backward pass): unnormalised, per-head or per-token decay
    if (a.normalize) return cudaErrorInvalidValue;
    if (a.g)
      return a.phi ? launch_cfg<DK, DVT, 64, NS, false, true, true, true>(a, workspace, stream, why)
                   : launch_cfg<DK, DVT, 64, NS, false, false, true, true>(a, workspace, stream, why);
    return a.phi ? launch_cfg<DK, DVT, 64, NS, false, true, false, true>(a, workspace, stream, why)
                 : launch_cfg<DK, DVT, 64, NS, false, false, false, true>(a, workspace, stream, why);
  }
  return a.g ? launch_shape_gated<DK, DVT, NS, true>(a, workspace, stream, why)
             : launch_shape_gated<DK, DVT, NS, false>(a, workspace, stream, why);
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, void *workspace, size_t, cudaStream_t stream, const char **why) {
  static_assert(tc_dvt(128) == 128 && tc_dvt(256) == 64, "value-slice widths");
  if (a.dk == 256) return launch_shape<256, 64, 2>(a, workspace, stream, why);
  return launch_shape<128, 128, 3>(a, workspace, stream, why);
}

}  // namespace la
