// la_bwd.cu -- backward of chunkwise causal linear attention (unnormalised,
// per-head decay), on CUDA cores with fp32 arithmetic.
//
// The forward of "1.6 长上下文与高效注意力", section 线性注意力, with the decay
// gamma: S_t = gamma S_{t-1} + v_t phi(k_t)^T, o_t = S_t phi(q_t).  For a loss
// with gradient dout_t at o_t:
//   dqh_t = S_t^T dout_t                           (forward in time)
//   G_t   = dout_t qh_t^T + gamma G_{t+1}          (backward in time)
//   dkh_t = G_t^T v_t,   dv_t = G_t kh_t,   dq = dqh phi'(q),  dk = dkh phi'(k).
// Regrouped into chunks of C' tokens (positions i, j inside the chunk):
//   dqh_i = sum_{j<=i} gamma^(i-j) (dout_i . v_j) kh_j + gamma^(i+1) S_p^T dout_i
//   dv_j  = sum_{i>=j} gamma^(i-j) (qh_i . kh_j) dout_i + gamma^(C'-j) R kh_j
//   dkh_j = sum_{i>=j} gamma^(i-j) (dout_i . v_j) qh_i  + gamma^(C'-j) R^T v_j
// with S_p the state before the chunk (carried forward as in the forward pass)
// and R = G at the next chunk's first token, carried backward:
//   R <- gamma^C' R + sum_i gamma^i dout_i qh_i^T.
// One CTA owns one (sequence, head): a forward sweep over its chunks writes dq,
// a backward sweep writes dk and dv.  S^T, then R^T, lives in shared memory
// ([d_k][d_v] fp32) next to the chunk's tiles; every product is fp32.
//
// Per-token decay (g set: alpha_t = exp(g_t), "1.6 长上下文与高效注意力", section
// 状态空间模型与 Mamba): with b_i the chunk's prefix sums of g, gamma^(i-j) becomes
// exp(b_i - b_j), gamma^(i+1) exp(b_i), and the state update's weights
// exp(b_last - b_j) and exp(b_last).  The backward carry is kept as
// Rt = alpha(next chunk's first token) R, so that
//   dv_j, dkh_j inter terms:  exp(b_last - b_j) Rt kh_j,  exp(b_last - b_j) Rt^T v_j
//   Rt <- exp(b_last) Rt + sum_i exp(b_i) dout_i qh_i^T
// (with b_i = (i + 1) ln gamma this is the per-head recursion above).  The loss
// sees b only through those weights, so dL/db_s = qh_s . dqh_s - kh_s . dkh_s;
// the sweeps add these row terms into dg (zeroed by the caller, fp32 atomics
// after a warp reduction) and a later kernel takes the reverse cumulative sum.
#include <cuda_bf16.h>

#include "la_common.cuh"
#include "la_internal.h"

namespace la {
namespace {

constexpr int kBwdThreads = 256;

struct BwdLayout {
  int C;
  size_t smem;
  int off_s, off_q, off_k, off_v, off_d, off_a, off_b, off_pw, off_bt;  // float offsets
};

BwdLayout bwd_layout(int dk, int dv, int C) {
  BwdLayout L;
  L.C = C;
  int o = 0;
  L.off_s = o; o += dk * (dv + 1);
  L.off_q = o; o += C * (dk + 1);
  L.off_k = o; o += C * (dk + 1);
  L.off_v = o; o += C * (dv + 1);
  L.off_d = o; o += C * (dv + 1);
  L.off_a = o; o += C * (C + 1);
  L.off_b = o; o += C * (C + 1);
  L.off_pw = o; o += C + 1;
  L.off_bt = o; o += C + 1;
  L.smem = (size_t)o * sizeof(float);
  return L;
}

// phi'(x) from phi(x) = ph: 1 for the identity; for elu + 1, 1 when x > 0 and
// e^x = ph otherwise, i.e. min(ph, 1) (ph > 1 exactly when x > 0).
__device__ __forceinline__ float dphi_from_phi(float ph, int phi) { return phi ? fminf(ph, 1.f) : 1.f; }

template <typename Tin>
__global__ void __launch_bounds__(kBwdThreads)
bwd_simt_kernel(BwdArgs a, BwdLayout L) {
  extern __shared__ float sm[];
  float *St = sm + L.off_s;    // [dk][dv+1] S^T in the forward sweep, R^T in the backward sweep
  float *qh = sm + L.off_q;    // [C][dk+1] phi(q) of the chunk
  float *kh = sm + L.off_k;    // [C][dk+1] phi(k)
  float *vv = sm + L.off_v;    // [C][dv+1] v
  float *dd = sm + L.off_d;    // [C][dv+1] dout
  float *A = sm + L.off_a;     // [C][C+1]  gamma^(i-j) dout_i . v_j   (j <= i)
  float *Bm = sm + L.off_b;    // [C][C+1]  gamma^(i-j) qh_i . kh_j    (j <= i)
  float *pw = sm + L.off_pw;   // [C+1]     gamma^n
  float *bt = sm + L.off_bt;   // [C]       per-token decay: prefix sums of g over the chunk

  const int tid = threadIdx.x;
  const int C = L.C, dk = a.dk, dv = a.dv;
  const int64_t unit = blockIdx.x;
  const int h = (int)(unit % a.H);
  const int64_t n = unit / a.H;
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
  const bool gated = a.g != nullptr;
  const float g = gated ? 1.f : a.gamma[h];
  const Tin *Q = (const Tin *)a.q.data + b * a.q.sb + h * a.q.sh;
  const Tin *K = (const Tin *)a.k.data + b * a.k.sb + h * a.k.sh;
  const Tin *V = (const Tin *)a.v.data + b * a.v.sb + h * a.v.sh;
  const Tin *D = (const Tin *)a.dout.data + b * a.dout.sb + h * a.dout.sh;
  Tin *DQ = (Tin *)a.dq.data + b * a.dq.sb + h * a.dq.sh;
  Tin *DK = (Tin *)a.dk_.data + b * a.dk_.sb + h * a.dk_.sh;
  Tin *DV = (Tin *)a.dv_.data + b * a.dv_.sb + h * a.dv_.sh;

  const int ds = dv + 1;  // padded row of S^T / R^T
  for (int e = tid; e < dk * ds; e += kBwdThreads) St[e] = 0.f;
  for (int i = tid; i <= C; i += kBwdThreads) pw[i] = decay_pow(g, i);

  // the chunk's phi(q), phi(k), v, dout (rows past the chunk end are zero)
  auto load_chunk = [&](int64_t c0, int Cp) {
    for (int e = tid; e < C * dk; e += kBwdThreads) {
      const int i = e / dk, c = e % dk;
      float x = 0.f, y = 0.f;
      if (i < Cp) {
        const int64_t t = start + c0 + i;
        x = feature_map(to_f32<Tin>(Q[t * a.q.st + c]), a.phi);
        y = feature_map(to_f32<Tin>(K[t * a.k.st + c]), a.phi);
      }
      qh[i * (dk + 1) + c] = x;
      kh[i * (dk + 1) + c] = y;
    }
    for (int e = tid; e < C * dv; e += kBwdThreads) {
      const int i = e / dv, r = e % dv;
      float x = 0.f, y = 0.f;
      if (i < Cp) {
        const int64_t t = start + c0 + i;
        x = to_f32<Tin>(V[t * a.v.st + r]);
        y = to_f32<Tin>(D[t * a.dout.st + r]);
      }
      vv[i * (dv + 1) + r] = x;
      dd[i * (dv + 1) + r] = y;
    }
  };
  // per-token decay: prefix sums b_i of the chunk's log decays (one thread; the
  // caller synchronises before use)
  auto load_decay = [&](int64_t c0, int Cp) {
    if (gated && tid == 0) {
      float acc = 0.f;
      const float *gp = a.g + (b * a.T + start + c0) * a.H + h;
      for (int i = 0; i < C; ++i) {
        if (i < Cp) acc += gp[(int64_t)i * a.H];
        bt[i] = acc;
      }
    }
  };
  // decay factors: D(i, j) = gamma^(i-j), E(i) = gamma^(i+1), W(j) = gamma^(Cp-1-j),
  // F(Cp) = gamma^Cp (per-token: differences of the prefix sums)
  auto Dij = [&](int i, int j) { return gated ? expf(bt[i] - bt[j]) : pw[i - j]; };
  auto Ei = [&](int i) { return gated ? expf(bt[i]) : pw[i + 1]; };
  auto Wj = [&](int j, int Cp) { return gated ? expf(bt[Cp - 1] - bt[j]) : pw[Cp - 1 - j]; };
  auto Fc = [&](int Cp) { return gated ? expf(bt[Cp - 1]) : pw[Cp]; };
  // decayed score tiles of the chunk (lower triangle, diagonal included)
  auto scores = [&](int Cp, bool with_b) {
    for (int e = tid; e < C * C; e += kBwdThreads) {
      const int i = e / C, j = e % C;
      float sa = 0.f, sb = 0.f;
      if (j <= i && i < Cp) {
        const float dij = Dij(i, j);
        const float *di = dd + i * (dv + 1), *vj = vv + j * (dv + 1);
        for (int r = 0; r < dv; ++r) sa = fmaf(di[r], vj[r], sa);
        sa *= dij;
        if (with_b) {
          const float *qi = qh + i * (dk + 1), *kj = kh + j * (dk + 1);
          for (int c = 0; c < dk; ++c) sb = fmaf(qi[c], kj[c], sb);
          sb *= dij;
        }
      }
      A[i * (C + 1) + j] = sa;
      if (with_b) Bm[i * (C + 1) + j] = sb;
    }
  };
  // dg row term x at row i of the chunk: reduced over the row's lanes (a row's d_k
  // elements are consecutive e; d_k >= 16 divides 32 or is a multiple of it), then
  // one atomic add per row.  Called by every thread with the same trip count.
  const int lane = tid & 31, rw = dk < 32 ? dk : 32;
  auto add_dg = [&](bool live, int64_t row, float x) {
    for (int o = rw / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (live && lane % rw == 0) atomicAdd(a.dg + (b * a.T + row) * a.H + h, x);
  };
  __syncthreads();

  // ---- forward sweep: dq
  for (int64_t c0 = 0; c0 < len; c0 += C) {
    const int Cp = (int)min((int64_t)C, len - c0);
    load_chunk(c0, Cp);
    load_decay(c0, Cp);
    __syncthreads();
    scores(Cp, false);
    __syncthreads();
    for (int e0 = 0; e0 < Cp * dk; e0 += kBwdThreads) {
      const int e = e0 + tid;
      const bool live = e < Cp * dk;
      const int i = live ? e / dk : 0, c = e % dk;
      float dqh = 0.f;
      if (live) {
        float intra = 0.f, inter = 0.f;
        for (int j = 0; j <= i; ++j) intra = fmaf(A[i * (C + 1) + j], kh[j * (dk + 1) + c], intra);
        const float *di = dd + i * (dv + 1), *sc = St + c * ds;
        for (int r = 0; r < dv; ++r) inter = fmaf(sc[r], di[r], inter);
        dqh = fmaf(Ei(i), inter, intra);
        DQ[(start + c0 + i) * a.dq.st + c] = from_f32<Tin>(dqh * dphi_from_phi(qh[i * (dk + 1) + c], a.phi));
      }
      if (gated) add_dg(live, start + c0 + i, qh[i * (dk + 1) + c] * dqh);
    }
    __syncthreads();
    // S^T <- gamma^C' S^T + sum_j gamma^(C'-1-j) kh_j v_j^T
    const float fc = Fc(Cp);
    for (int e = tid; e < dk * dv; e += kBwdThreads) {
      const int c = e / dv, r = e % dv;
      float acc = 0.f;
      for (int j = 0; j < Cp; ++j) acc = fmaf(Wj(j, Cp) * kh[j * (dk + 1) + c], vv[j * (dv + 1) + r], acc);
      St[c * ds + r] = fmaf(fc, St[c * ds + r], acc);
    }
    __syncthreads();
  }

  // ---- backward sweep: dk, dv (St holds R^T, starting at zero)
  for (int e = tid; e < dk * ds; e += kBwdThreads) St[e] = 0.f;
  const int64_t nch = (len + C - 1) / C;
  for (int64_t ci = nch - 1; ci >= 0; --ci) {
    const int64_t c0 = ci * C;
    const int Cp = (int)min((int64_t)C, len - c0);
    __syncthreads();
    load_chunk(c0, Cp);
    load_decay(c0, Cp);
    __syncthreads();
    scores(Cp, true);
    __syncthreads();
    // inter-chunk weight of row j: gamma^(C'-j) on R (per-token: exp(b_last - b_j) on Rt)
    auto Ij = [&](int j) { return gated ? expf(bt[Cp - 1] - bt[j]) : pw[Cp - j]; };
    // dv_j = sum_{i>=j} B_ij dout_i + gamma^(C'-j) R kh_j
    for (int e = tid; e < Cp * dv; e += kBwdThreads) {
      const int j = e / dv, r = e % dv;
      float intra = 0.f, inter = 0.f;
      for (int i = j; i < Cp; ++i) intra = fmaf(Bm[i * (C + 1) + j], dd[i * (dv + 1) + r], intra);
      const float *kj = kh + j * (dk + 1);
      for (int c = 0; c < dk; ++c) inter = fmaf(St[c * ds + r], kj[c], inter);
      DV[(start + c0 + j) * a.dv_.st + r] = from_f32<Tin>(fmaf(Ij(j), inter, intra));
    }
    // dkh_j = sum_{i>=j} A_ij qh_i + gamma^(C'-j) R^T v_j
    for (int e0 = 0; e0 < Cp * dk; e0 += kBwdThreads) {
      const int e = e0 + tid;
      const bool live = e < Cp * dk;
      const int j = live ? e / dk : 0, c = e % dk;
      float dkh = 0.f;
      if (live) {
        float intra = 0.f, inter = 0.f;
        for (int i = j; i < Cp; ++i) intra = fmaf(A[i * (C + 1) + j], qh[i * (dk + 1) + c], intra);
        const float *vj = vv + j * (dv + 1), *sc = St + c * ds;
        for (int r = 0; r < dv; ++r) inter = fmaf(sc[r], vj[r], inter);
        dkh = fmaf(Ij(j), inter, intra);
        DK[(start + c0 + j) * a.dk_.st + c] = from_f32<Tin>(dkh * dphi_from_phi(kh[j * (dk + 1) + c], a.phi));
      }
      if (gated) add_dg(live, start + c0 + j, -kh[j * (dk + 1) + c] * dkh);
    }
    __syncthreads();
    // R^T <- gamma^C' R^T + sum_i gamma^i qh_i dout_i^T
    // (per-token: Rt^T <- exp(b_last) Rt^T + sum_i exp(b_i) qh_i dout_i^T)
    const float fc = Fc(Cp);
    for (int e = tid; e < dk * dv; e += kBwdThreads) {
      const int c = e / dv, r = e % dv;
      float acc = 0.f;
      for (int i = 0; i < Cp; ++i)
        acc = fmaf((gated ? expf(bt[i]) : pw[i]) * qh[i * (dk + 1) + c], dd[i * (dv + 1) + r], acc);
      St[c * ds + r] = fmaf(fc, St[c * ds + r], acc);
    }
  }
}

bool pick_bwd_layout(const BwdArgs &a, int device, BwdLayout *out) {
  const int limit = max_smem_optin(device);
  for (int C : {a.chunk, 64, 32, 16}) {
    if (C > a.chunk) continue;
    BwdLayout L = bwd_layout(a.dk, a.dv, C);
    if ((int64_t)L.smem <= limit) {
      *out = L;
      return true;
    }
  }
  return false;
}

}  // namespace

bool bwd_supported(const BwdArgs &a, int device) {
  BwdLayout L;
  return pick_bwd_layout(a, device, &L);
}

cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t stream) {
  int device = 0;
  cudaError_t err = cudaGetDevice(&device);
  if (err != cudaSuccess) return err;
  BwdLayout L;
  if (!pick_bwd_layout(a, device, &L)) return cudaErrorInvalidConfiguration;
  const int64_t grid = a.n_seqs * a.H;
  if (grid == 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (a.dtype == LA_F32) {
    auto kern = bwd_simt_kernel<float>;
    if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem)) != cudaSuccess)
      return err;
    kern<<<(unsigned)grid, kBwdThreads, L.smem, stream>>>(a, L);
  } else {
    auto kern = bwd_simt_kernel<__nv_bfloat16>;
    if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem)) != cudaSuccess)
      return err;
    kern<<<(unsigned)grid, kBwdThreads, L.smem, stream>>>(a, L);
  }
  return cudaGetLastError();
}

}  // namespace la
