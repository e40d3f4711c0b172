// la_simt.cu -- chunkwise causal linear attention forward on CUDA cores, fp32.
//
// The chunk form follows from unrolling the recurrence of "1.6 长上下文与高效注意力",
// section 线性注意力 (S_t = gamma S_{t-1} + v_t phi(k_t)^T, o_t = S_t phi(q_t), the
// optional normaliser z_t) from the state S_p that the first token of a chunk
// sees.  For positions i, j < C' in a chunk of C' tokens:
//   o_i   = gamma^(i+1) S_p qh_i + sum_{j<=i} gamma^(i-j) (qh_i . kh_j) v_j
//   den_i = gamma^(i+1) z_p . qh_i + sum_{j<=i} gamma^(i-j) (qh_i . kh_j)
//   S'    = gamma^C' S_p + sum_j gamma^(C'-1-j) v_j kh_j^T     (z' likewise)
// With a data-dependent decay alpha_t = exp(g_t) (section 状态空间模型与 Mamba)
// every gamma^n above becomes a product of the alphas it spans: with the chunk's
// prefix sums b_i = sum_{t<=i} g_t, gamma^(i-j) -> exp(b_i - b_j), gamma^(i+1) ->
// exp(b_i), gamma^C' -> exp(b_{C'-1}) and gamma^(C'-1-j) -> exp(b_{C'-1} - b_j).
// This kernel is the exact-arithmetic path: f32 inputs (no TF32 anywhere) and
// any shape the tensor-core kernel does not take.  One CTA owns one
// (sequence, head, slice of d_v columns) and walks its chunks in order, with
// S^T[:, slice] and z resident in shared memory.
#include <cuda_bf16.h>

#include "la_common.cuh"
#include "la_internal.h"

namespace la {
namespace {

constexpr int kSimtThreads = 256;

struct SimtLayout {
  int dvt;  // d_v columns per CTA
  int n_vt;
  size_t smem;
  // float offsets
  int off_st, off_z, off_q, off_k, off_v, off_p, off_pw, off_den, off_b;
};

SimtLayout simt_layout(int dk, int dv, int C, int dvt) {
  SimtLayout L;
  L.dvt = dvt;
  L.n_vt = (dv + dvt - 1) / dvt;
  int o = 0;
  L.off_st = o; o += dk * dvt;
  L.off_z = o; o += dk;
  L.off_q = o; o += C * (dk + 1);
  L.off_k = o; o += C * (dk + 1);
  L.off_v = o; o += C * dvt;
  L.off_p = o; o += C * (C + 1);
  L.off_pw = o; o += C + 1;
  L.off_den = o; o += C;
  L.off_b = o; o += C;
  L.smem = (size_t)o * sizeof(float);
  return L;
}

bool pick_layout(const ChunkArgs &a, int device, SimtLayout *out) {
  const int limit = max_smem_optin(device);
  for (int dvt : {64, 32, 16}) {
    SimtLayout L = simt_layout(a.dk, a.dv, a.chunk, dvt < a.dv ? dvt : a.dv);
    if ((int64_t)L.smem <= limit) {
      *out = L;
      return true;
    }
  }
  return false;
}

template <typename Tin>
__global__ void __launch_bounds__(kSimtThreads)
chunk_simt_kernel(ChunkArgs a, SimtLayout L) {
  extern __shared__ float sm[];
  float *St = sm + L.off_st;    // [dk][dvt]   S^T restricted to this CTA's columns
  float *z = sm + L.off_z;      // [dk]
  float *qh = sm + L.off_q;     // [C][dk+1]   phi(q) of the chunk
  float *kh = sm + L.off_k;     // [C][dk+1]   phi(k)
  float *vv = sm + L.off_v;     // [C][dvt]
  float *P = sm + L.off_p;      // [C][C+1]    decay-masked scores
  float *pw = sm + L.off_pw;    // [C+1]       gamma^n
  float *den = sm + L.off_den;  // [C]
  float *bsum = sm + L.off_b;   // [C]         data-dependent decay: chunk prefix sums of g

  const int tid = threadIdx.x;
  const int C = a.chunk, dk = a.dk, dvt = L.dvt;
  const int64_t unit = blockIdx.x;
  const int vt = (int)(unit % L.n_vt);
  const int h = (int)((unit / L.n_vt) % a.H);
  const int64_t n = unit / ((int64_t)L.n_vt * a.H);
  const int v0 = vt * dvt;
  const int ncols = min(dvt, a.dv - v0);

  int64_t b, start, len;
  if (a.cu_seqlens) {
    b = 0;
    start = a.cu_seqlens[n];
    len = (int64_t)a.cu_seqlens[n + 1] - start;
  } else {
    b = n;
    start = 0;
    len = a.T;
  }
  const float g = a.g ? 1.f : a.gamma[h];
  const bool gated = a.g != nullptr;
  const Tin *Q = (const Tin *)a.q.data + b * a.q.sb + h * a.q.sh;
  const Tin *K = (const Tin *)a.k.data + b * a.k.sb + h * a.k.sh;
  const Tin *V = (const Tin *)a.v.data + b * a.v.sb + h * a.v.sh + v0;
  Tin *O = (Tin *)a.out + b * a.o_sb + h * a.o_sh + v0;

  for (int i = tid; i < dk * dvt; i += kSimtThreads) St[i] = 0.f;
  for (int i = tid; i < dk; i += kSimtThreads) z[i] = 0.f;
  for (int i = tid; i <= C; i += kSimtThreads) pw[i] = decay_pow(g, i);
  __syncthreads();

  for (int64_t c0 = 0; c0 < len; c0 += C) {
    const int Cp = (int)min((int64_t)C, len - c0);
    // ---- load phi(q), phi(k), v of the chunk (rows >= Cp are zero)
    for (int e = tid; e < C * dk; e += kSimtThreads) {
      const int i = e / dk, c = e % dk;
      float qv = 0.f, kv = 0.f;
      if (i < Cp) {
        const int64_t t = start + c0 + i;
        qv = feature_map(to_f32<Tin>(Q[t * a.q.st + c]), a.phi);
        kv = feature_map(to_f32<Tin>(K[t * a.k.st + c]), a.phi);
      }
      qh[i * (dk + 1) + c] = qv;
      kh[i * (dk + 1) + c] = kv;
    }
    for (int e = tid; e < C * dvt; e += kSimtThreads) {
      const int i = e / dvt, r = e % dvt;
      float x = 0.f;
      if (i < Cp && r < ncols) x = to_f32<Tin>(V[(start + c0 + i) * a.v.st + r]);
      vv[e] = x;
    }
    if (gated && tid == 0) {  // prefix sums of the log decay over the chunk
      float acc = 0.f;
      const float *gp = a.g + (b * a.T + start + c0) * a.H + h;
      for (int i = 0; i < C; ++i) {
        if (i < Cp) acc += gp[(int64_t)i * a.H];
        bsum[i] = acc;
      }
    }
    __syncthreads();
    // decay factors of the chunk: D(i, j) = gamma^(i-j), E(i) = gamma^(i+1),
    // W(j) = gamma^(Cp-1-j) (data-dependent: differences of the prefix sums)
    auto Dij = [&](int i, int j) { return gated ? expf(bsum[i] - bsum[j]) : pw[i - j]; };
    auto Ei = [&](int i) { return gated ? expf(bsum[i]) : pw[i + 1]; };
    auto Wj = [&](int j) { return gated ? expf(bsum[Cp - 1] - bsum[j]) : pw[Cp - 1 - j]; };
    // ---- P = (qh kh^T) * D, D_ij = gamma^(i-j) for j <= i (diagonal kept)
    for (int e = tid; e < C * C; e += kSimtThreads) {
      const int i = e / C, j = e % C;
      float acc = 0.f;
      if (j <= i && i < Cp) {
        const float *qi = qh + i * (dk + 1);
        const float *kj = kh + j * (dk + 1);
        for (int c = 0; c < dk; ++c) acc = fmaf(qi[c], kj[c], acc);
        acc *= Dij(i, j);
      }
      P[i * (C + 1) + j] = acc;
    }
    __syncthreads();
    // ---- denominators: gamma^(i+1) z.qh_i + row sum of P
    if (a.normalize) {
      for (int i = tid; i < C; i += kSimtThreads) {
        float zq = 0.f, ps = 0.f;
        const float *qi = qh + i * (dk + 1);
        for (int c = 0; c < dk; ++c) zq = fmaf(z[c], qi[c], zq);
        for (int j = 0; j <= i; ++j) ps += P[i * (C + 1) + j];
        den[i] = fmaf(Ei(i), zq, ps);
      }
      __syncthreads();
    }
    // ---- outputs: gamma^(i+1) qh_i S_p^T + P V
    for (int e = tid; e < Cp * dvt; e += kSimtThreads) {
      const int i = e / dvt, r = e % dvt;
      if (r >= ncols) continue;
      const float *qi = qh + i * (dk + 1);
      float inter = 0.f, intra = 0.f;
      for (int c = 0; c < dk; ++c) inter = fmaf(qi[c], St[c * dvt + r], inter);
      for (int j = 0; j <= i; ++j) intra = fmaf(P[i * (C + 1) + j], vv[j * dvt + r], intra);
      float o = fmaf(Ei(i), inter, intra);
      if (a.normalize) o = o / den[i];
      O[(start + c0 + i) * a.o_st + r] = from_f32<Tin>(o);
    }
    __syncthreads();
    // ---- carry: S^T <- gamma^Cp S^T + sum_j gamma^(Cp-1-j) kh_j v_j^T ; z likewise
    const float gC = gated ? expf(bsum[Cp - 1]) : pw[Cp];
    for (int e = tid; e < dk * dvt; e += kSimtThreads) {
      const int c = e / dvt, r = e % dvt;
      float acc = 0.f;
      for (int j = 0; j < Cp; ++j) acc = fmaf(Wj(j) * kh[j * (dk + 1) + c], vv[j * dvt + r], acc);
      St[e] = fmaf(gC, St[e], acc);
    }
    if (a.normalize) {
      for (int c = tid; c < dk; c += kSimtThreads) {
        float acc = 0.f;
        for (int j = 0; j < Cp; ++j) acc = fmaf(Wj(j), kh[j * (dk + 1) + c], acc);
        z[c] = fmaf(gC, z[c], acc);
      }
    }
    __syncthreads();
  }

  if (a.final_z && v0 == 0) {  // z after the last token (kept only when normalising)
    float *Zf = a.final_z + ((int64_t)n * a.H + h) * (int64_t)dk;
    for (int c = tid; c < dk; c += kSimtThreads) Zf[c] = z[c];
  }
  if (a.final_state) {
    float *F = a.final_state + ((int64_t)n * a.H + h) * (int64_t)dk * a.dv + v0;
    for (int e = tid; e < dk * dvt; e += kSimtThreads) {
      const int c = e / dvt, r = e % dvt;
      if (r < ncols) F[(int64_t)c * a.dv + r] = St[e];
    }
  }
}

}  // namespace

bool simt_supported(const ChunkArgs &a, int device) {
  SimtLayout L;
  return pick_layout(a, device, &L);
}

cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream) {
  int device = 0;
  cudaError_t err = cudaGetDevice(&device);
  if (err != cudaSuccess) return err;
  SimtLayout L;
  if (!pick_layout(a, device, &L)) return cudaErrorInvalidConfiguration;
  const int64_t grid = a.n_seqs * a.H * L.n_vt;
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (a.dtype == LA_F32) {
    err = cudaFuncSetAttribute(chunk_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)L.smem);
    if (err != cudaSuccess) return err;
    chunk_simt_kernel<float><<<(unsigned)grid, kSimtThreads, L.smem, stream>>>(a, L);
  } else {
    err = cudaFuncSetAttribute(chunk_simt_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
    if (err != cudaSuccess) return err;
    chunk_simt_kernel<__nv_bfloat16><<<(unsigned)grid, kSimtThreads, L.smem, stream>>>(a, L);
  }
  return cudaGetLastError();
}

}  // namespace la
