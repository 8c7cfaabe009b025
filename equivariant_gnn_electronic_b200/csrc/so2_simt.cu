// CUDA-core (SIMT) eSCN layer and Hamiltonian head: one CTA per destination atom,
// the atom's incoming edges in chunks of `te`.  Exact fp32 arithmetic (no TF32),
// bf16 or fp32 storage.  This is the path of the fp32 workload and the fallback
// for shapes the tensor-core kernel does not take; its reads of the weights
// (every chunk re-reads them from L2) make it far slower than that kernel.
//
// Method: "MALOQ: Massively Accelerated Learning of Operators for Quantum
// Transport", Sections II-B1 and III (rotate each edge onto one axis, SO(2)
// constrained linear layers, aggregate onto the target), Section III-D and
// Fig. 4(b) (message from the concatenated pair), Section III-B1 Eq. (1)
// (Clebsch-Gordan map from labels to orbital blocks); the review page of
// "Distributed Equivariant Graph Neural Networks for Large-Scale Electronic
// Structure Prediction", "What carries the argument" (attention and
// aggregation local to the atom that owns the incoming edges).
#include <math.h>

#include "common.cuh"
#include "so2_params.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxTE = 8;

struct Smem {
  float *nd, *acc, *D, *rb, *hid, *gate, *X, *Y, *lg, *p, *st;
  int* srcs;
};

__device__ __forceinline__ Smem carve(float* base, const So2Params& P, int te) {
  Smem s;
  float* q = base;
  s.nd = q;   q += P.L2 * P.C;
  s.acc = q;  q += P.L2 * P.C;
  s.D = q;    q += te * P.wfl;
  s.rb = q;   q += te * P.K;
  s.hid = q;  q += te * P.C;
  s.gate = q; q += te * P.L * 2 * P.C;
  s.X = q;    q += te * P.nrows * 2 * P.C;
  s.Y = q;    q += te * P.nrows * P.C;
  s.lg = q;   q += te * P.H;
  s.p = q;    q += te * P.H;
  s.st = q;   q += 4 * P.H;      // running max, running sum, scale, spare
  s.srcs = (int*)q;
  return s;
}

// Gate, rotate-in, SO(2) linear for edges [e0, e0+ne) of destination d (into s.Y).
template <typename T>
__device__ void so2_chunk(const So2Params& P, const So2Weights& W, const Smem& s, int d, int e0,
                          int ne) {
  const T* nin = (const T*)P.node_in;
  const int C = P.C, C2 = 2 * P.C, L = P.L, K = P.K;
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int i = tid; i < ne; i += nt) {
    int sidx = P.src[e0 + i];
    if (sidx < 0 || sidx >= P.n_atoms) {
      egnn_flag(P.status, EGNN_DEV_INDEX_RANGE);
      sidx = d;
    }
    s.srcs[i] = sidx;
  }
  for (int i = tid; i < ne * P.wfl; i += nt) {
    int e = i / P.wfl, j = i - e * P.wfl;
    s.D[e * P.wfl + j] = P.wig[(long long)(e0 + e) * P.wfl + j];
  }
  const float mu_step = P.rcut / (float)(K - 1);
  const float inv2s2 = 1.0f / (2.0f * mu_step * mu_step);
  for (int i = tid; i < ne * K; i += nt) {
    int e = i / K, k = i - e * K;
    float dd = P.dist[e0 + e] - k * mu_step;
    s.rb[e * K + k] = expf(-dd * dd * inv2s2);
  }
  __syncthreads();
  const T* W1 = (const T*)W.W1;
  const T* b1 = (const T*)W.b1;
  for (int i = tid; i < ne * C; i += nt) {
    int e = i / C, c = i - e * C;
    float a = egnn_ld(b1, c);
    for (int k = 0; k < K; ++k) a += egnn_ld(W1, (long long)c * K + k) * s.rb[e * K + k];
    s.hid[e * C + c] = a / (1.0f + expf(-a));
  }
  __syncthreads();
  const T* W2 = (const T*)W.W2;
  const T* b2 = (const T*)W.b2;
  for (int j = tid; j < L * C2; j += nt) {
    float acc[kMaxTE];
    float bj = egnn_ld(b2, j);
    for (int e = 0; e < kMaxTE; ++e) acc[e] = bj;
    for (int c = 0; c < C; ++c) {
      float w = egnn_ld(W2, (long long)j * C + c);
#pragma unroll
      for (int e = 0; e < kMaxTE; ++e)
        if (e < ne) acc[e] += w * s.hid[e * C + c];
    }
    for (int e = 0; e < ne; ++e) s.gate[e * L * C2 + j] = acc[e];
  }
  __syncthreads();
  // rotate into the edge frame, keep |m| <= mmax, gate: X[e][row][c2]
  for (int i = tid; i < P.nrows * C2; i += nt) {
    int r = i / C2, c2 = i - r * C2;
    int l = P.row_l[r], m = P.row_m[r];
    int ml = l < P.mmax ? l : P.mmax;
    int dl = 2 * l + 1;
    int wo = P.woff[l] + (m + ml) * dl;
    for (int e = 0; e < ne; ++e) {
      const float* Dr = s.D + e * P.wfl + wo;
      float a = 0.f;
      if (c2 < C) {
        const T* z = nin + ((long long)s.srcs[e] * P.L2 + l * l) * C + c2;
        for (int mp = 0; mp < dl; ++mp) a += Dr[mp] * egnn_ld(z, (long long)mp * C);
      } else {
        const float* z = s.nd + l * l * C + (c2 - C);
        for (int mp = 0; mp < dl; ++mp) a += Dr[mp] * z[mp * C];
      }
      s.X[(e * P.nrows + r) * C2 + c2] = a * s.gate[e * L * C2 + l * C2 + c2];
    }
  }
  __syncthreads();
  // SO(2) linear; one warp per output row, lanes split the reduction
  const int warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
  const T* W0 = (const T*)W.W0;
  for (int o = warp; o < L * C; o += nw) {
    float acc[kMaxTE];
    for (int e = 0; e < kMaxTE; ++e) acc[e] = 0.f;
    for (int k = lane; k < L * C2; k += 32) {
      float w = egnn_ld(W0, (long long)o * L * C2 + k);
      int l = k / C2, c2 = k - l * C2;
      int r = P.row0[l];
#pragma unroll
      for (int e = 0; e < kMaxTE; ++e)
        if (e < ne) acc[e] += w * s.X[(e * P.nrows + r) * C2 + c2];
    }
    int lo = o / C, c = o - lo * C;
    for (int e = 0; e < ne; ++e) {
      float v = acc[e];
      for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) s.Y[(e * P.nrows + P.row0[lo]) * C + c] = v;
    }
  }
  for (int m = 1; m <= P.mmax; ++m) {
    const T* Wa = (const T*)W.Wm[m - 1][0];
    const T* Wb = (const T*)W.Wm[m - 1][1];
    const int nm = L - m;
    for (int o = warp; o < nm * C; o += nw) {
      float ap[kMaxTE], am[kMaxTE];
      for (int e = 0; e < kMaxTE; ++e) ap[e] = am[e] = 0.f;
      for (int k = lane; k < nm * C2; k += 32) {
        float wa = egnn_ld(Wa, (long long)o * nm * C2 + k);
        float wb = egnn_ld(Wb, (long long)o * nm * C2 + k);
        int i = k / C2, c2 = k - i * C2;
        int l = m + i;
        int rp = P.row0[l] + m, rm = P.row0[l] - m;
#pragma unroll
        for (int e = 0; e < kMaxTE; ++e)
          if (e < ne) {
            float xp = s.X[(e * P.nrows + rp) * C2 + c2];
            float xm = s.X[(e * P.nrows + rm) * C2 + c2];
            ap[e] += wa * xp - wb * xm;
            am[e] += wb * xp + wa * xm;
          }
      }
      int i = o / C, c = o - i * C;
      int l = m + i;
      for (int e = 0; e < ne; ++e) {
        float vp = ap[e], vm = am[e];
        for (int off = 16; off; off >>= 1) {
          vp += __shfl_xor_sync(0xffffffffu, vp, off);
          vm += __shfl_xor_sync(0xffffffffu, vm, off);
        }
        if (lane == 0) {
          s.Y[(e * P.nrows + P.row0[l] + m) * C + c] = vp;
          s.Y[(e * P.nrows + P.row0[l] - m) * C + c] = vm;
        }
      }
    }
  }
  __syncthreads();
}

// msg[l, m', c] of edge e (rotate back with the kept rows of D^l)
__device__ __forceinline__ float rotate_back(const So2Params& P, const Smem& s, int e, int l, int mp,
                                             int c) {
  int ml = l < P.mmax ? l : P.mmax;
  int dl = 2 * l + 1;
  const float* Dl = s.D + e * P.wfl + P.woff[l];
  const float* Y = s.Y + (e * P.nrows + P.row0[l]) * P.C + c;
  float v = 0.f;
  for (int m = -ml; m <= ml; ++m) v += Dl[(m + ml) * dl + (mp + l)] * Y[m * P.C];
  return v;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) layer_simt_kernel(So2Params P, So2Weights W) {
  extern __shared__ float smem[];
  const int d = blockIdx.x;
  const int te = P.te;
  Smem s = carve(smem, P, te);
  const T* nin = (const T*)P.node_in;
  T* nout = (T*)P.node_out;
  const int C = P.C, tid = threadIdx.x, nt = blockDim.x;
  const int n_out = P.L2 * C;
  for (int i = tid; i < n_out; i += nt) {
    s.nd[i] = egnn_ld(nin, (long long)d * n_out + i);
    s.acc[i] = 0.f;
  }
  if (tid < P.H) {
    s.st[tid] = -INFINITY;
    s.st[P.H + tid] = 0.f;
  }
  int e_begin = P.row_ptr[d], e_end = P.row_ptr[d + 1];
  if (e_begin < 0 || e_end < e_begin || (long long)e_end > P.n_edges) {
    if (tid == 0) egnn_flag(P.status, EGNN_DEV_BAD_GRAPH);
    e_end = e_begin;
  }
  __syncthreads();
  const int hc = C / P.H;
  const T* A = (const T*)W.A;
  const T* bA = (const T*)W.bA;
  for (int e0 = e_begin; e0 < e_end; e0 += te) {
    int ne = min(te, e_end - e0);
    so2_chunk<T>(P, W, s, d, e0, ne);
    // attention logits from SiLU(y0): one warp per (edge, head)
    const int warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
    for (int q = warp; q < ne * P.H; q += nw) {
      int e = q / P.H, h = q - e * P.H;
      float a = 0.f;
      for (int j = lane; j < P.L * C; j += 32) {
        int l = j / C, c = j - l * C;
        float y = s.Y[(e * P.nrows + P.row0[l]) * C + c];
        a += egnn_ld(A, (long long)h * P.L * C + j) * (y / (1.0f + expf(-y)));
      }
      for (int off = 16; off; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0) s.lg[e * P.H + h] = a + egnn_ld(bA, h);
    }
    __syncthreads();
    if (tid < P.H) {   // online softmax state per head
      int h = tid;
      float mo = s.st[h], mn = mo;
      for (int e = 0; e < ne; ++e) mn = fmaxf(mn, s.lg[e * P.H + h]);
      float sc = (mo == -INFINITY) ? 0.f : expf(mo - mn);
      float sum = s.st[P.H + h] * sc;
      for (int e = 0; e < ne; ++e) {
        float pe = expf(s.lg[e * P.H + h] - mn);
        s.p[e * P.H + h] = pe;
        sum += pe;
      }
      s.st[h] = mn;
      s.st[P.H + h] = sum;
      s.st[2 * P.H + h] = sc;
    }
    __syncthreads();
    for (int i = tid; i < n_out; i += nt) {
      int lm = i / C, c = i - lm * C;
      int l = P.coef_l[lm], mp = lm - l * l - l;
      int h = c / hc;
      float a = s.acc[i] * s.st[2 * P.H + h];
      for (int e = 0; e < ne; ++e) a += s.p[e * P.H + h] * rotate_back(P, s, e, l, mp, c);
      s.acc[i] = a;
    }
    __syncthreads();
  }
  for (int i = tid; i < n_out; i += nt) {
    int c = i % C;
    int h = c / hc;
    float v = s.nd[i];
    if (e_end > e_begin) v += s.acc[i] / s.st[P.H + h];
    egnn_st(nout, (long long)d * n_out + i, v);
  }
}

// Hamiltonian head: per edge t = rotated-back SO(2) message, labels, CG -> block.
template <typename T>
__global__ void __launch_bounds__(kThreads) head_simt_kernel(So2Params P, So2Weights W, HeadTables Tb) {
  extern __shared__ float smem[];
  const int d = blockIdx.x;
  const int te = P.te;
  Smem s = carve(smem, P, te);
  const T* nin = (const T*)P.node_in;
  const int C = P.C, tid = threadIdx.x, nt = blockDim.x;
  const int n_emb = P.L2 * C;
  for (int i = tid; i < n_emb; i += nt) s.nd[i] = egnn_ld(nin, (long long)d * n_emb + i);
  int e_begin = P.row_ptr[d], e_end = P.row_ptr[d + 1];
  if (e_begin < 0 || e_end < e_begin || (long long)e_end > P.n_edges) {
    if (tid == 0) egnn_flag(P.status, EGNN_DEV_BAD_GRAPH);
    e_end = e_begin;
  }
  __syncthreads();
  float* Tm = s.X;      // t[e][L^2][C] reuses the rotated-input buffer
  float* lab = s.gate;  // labels[e][n_lab] reuse the gate buffer
  const int norb = Tb.n_orb, nlab = Tb.n_lab;
  for (int e0 = e_begin; e0 < e_end; e0 += te) {
    int ne = min(te, e_end - e0);
    so2_chunk<T>(P, W, s, d, e0, ne);
    for (int i = tid; i < ne * n_emb; i += nt) {
      int e = i / n_emb, r = i - e * n_emb;
      int lm = r / C, c = r - lm * C;
      int l = P.coef_l[lm], mp = lm - l * l - l;
      Tm[i] = rotate_back(P, s, e, l, mp, c);
    }
    __syncthreads();
    // labels: h[L][M][k] = sum_c U^L[k][c] t[L,M,c], stored at lab_off[L] + (M+L)*mult_L + k
    for (int i = tid; i < ne * nlab; i += nt) {
      int e = i / nlab, q = i - e * nlab;
      int Lq = 0;
      while (Lq + 1 <= P.lmax && Tb.lab_off[Lq + 1] <= q) ++Lq;
      int mult = Tb.mult[Lq];
      int r = q - Tb.lab_off[Lq];
      int M = r / mult, k = r - M * mult;
      const T* U = (const T*)W.U[Lq];
      const float* t = Tm + (long long)e * n_emb + (Lq * Lq + M) * C;
      float a = 0.f;
      for (int c = 0; c < C; ++c) a += egnn_ld(U, (long long)k * C + c) * t[c];
      lab[e * nlab + q] = a;
    }
    __syncthreads();
    // blocks: each entry sums its Clebsch-Gordan terms
    for (int i = tid; i < ne * norb * norb; i += nt) {
      int e = i / (norb * norb), q = i - e * norb * norb;
      int ri = q / norb, cj = q - ri * norb;
      int a = Tb.orb_shell[ri], b = Tb.orb_shell[cj];
      int la = Tb.shell_l[a], lb = Tb.shell_l[b];
      int ia = ri - Tb.shell_off[a], jb = cj - Tb.shell_off[b];
      float v = 0.f;
      for (int Lc = (la > lb ? la - lb : lb - la); Lc <= la + lb; ++Lc) {
        int k = Tb.kidx[(a * Tb.n_shells + b) * 8 + Lc];
        const float* cgm = Tb.cg + Tb.cg_off[(la * 4 + lb) * 8 + Lc] + (ia * (2 * lb + 1) + jb) * (2 * Lc + 1);
        const float* h = lab + e * nlab + Tb.lab_off[Lc] + k;
        int mult = Tb.mult[Lc];
        for (int M = 0; M < 2 * Lc + 1; ++M) v += cgm[M] * h[M * mult];
      }
      P.blocks[(long long)(e0 + e) * norb * norb + q] = v;
    }
    __syncthreads();
  }
}

}  // namespace

size_t so2_simt_smem_bytes(const So2Params& P, int te) {
  size_t f = 2 * (size_t)P.L2 * P.C + (size_t)te * (P.wfl + P.K + P.C + P.L * 2 * P.C + P.nrows * 2 * P.C +
                                                     P.nrows * P.C + 2 * P.H) + 4 * P.H;
  return f * sizeof(float) + (size_t)te * sizeof(int) + 16;
}

int so2_simt_pick_te(const So2Params& P, int head_labels) {
  int best = 0;
  for (int te = 1; te <= kMaxTE; ++te) {
    if (so2_simt_smem_bytes(P, te) > 200 * 1024) break;
    if (head_labels > 0 && head_labels > P.L * 2 * P.C) break;
    best = te;
  }
  return best;
}

cudaError_t launch_layer_simt(So2Params P, So2Weights W, cudaStream_t st) {
  size_t sm = so2_simt_smem_bytes(P, P.te);
  if (P.dtype == EGNN_FP32) {
    cudaFuncSetAttribute(layer_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    layer_simt_kernel<float><<<P.n_atoms, kThreads, sm, st>>>(P, W);
  } else {
    cudaFuncSetAttribute(layer_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    layer_simt_kernel<__nv_bfloat16><<<P.n_atoms, kThreads, sm, st>>>(P, W);
  }
  return cudaGetLastError();
}

cudaError_t launch_head_simt(So2Params P, So2Weights W, HeadTables T, cudaStream_t st) {
  size_t sm = so2_simt_smem_bytes(P, P.te);
  if (P.dtype == EGNN_FP32) {
    cudaFuncSetAttribute(head_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    head_simt_kernel<float><<<P.n_atoms, kThreads, sm, st>>>(P, W, T);
  } else {
    cudaFuncSetAttribute(head_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    head_simt_kernel<__nv_bfloat16><<<P.n_atoms, kThreads, sm, st>>>(P, W, T);
  }
  return cudaGetLastError();
}
