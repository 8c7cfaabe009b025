// Label <-> block conversion of orbital blocks, and assembly of the Hamiltonian.
//
// "MALOQ: Massively Accelerated Learning of Operators for Quantum Transport",
// Section III-B1 and Eq. (1): an orbital block H^{ab} of size (2l_a+1) x (2l_b+1)
// is the Clebsch-Gordan image of labels |L, M>, L = |l_a - l_b| .. l_a + l_b, and
// the labels are the projection of the block (the coupling matrices have
// orthonormal columns).  Section III-B2 and Fig. 2(b-d): the conversion runs on the
// GPU driven by the orbital template, one thread block per node or edge and one
// thread per matrix element; Label -> Matrix rebuilds the whole Hamiltonian.  The
// review page of "Distributed Equivariant Graph Neural Networks for Large-Scale
// Electronic Structure Prediction" gives the target: one matrix of 104,833 orbitals
// for the 8,064-atom GeSbTe cell.
//
// Kernels:
//   labels_to_blocks  CTA per group of blocks; labels staged in shared memory; one
//                     thread per matrix element sums its pair's labels through C^L.
//   blocks_to_labels  CTA per group of blocks; blocks staged in shared memory; one
//                     thread per label sums its pair's block through C^L.
//   h_count / h_scan / h_fill  block-sparse rows of the k = 0 Hamiltonian: row block d
//                     holds the on-site block of d and, per distinct source atom s of
//                     d's incoming edges, the sum of those edges' blocks (periodic
//                     images of one pair add up), column blocks ascending.
#include <math.h>
#include <string.h>

#include <vector>

#include "common.cuh"
#include "so2_params.cuh"

namespace {

constexpr int kLabLmax = 6;   // labels up to L = 2 * 3 (shells up to f)

struct LabelTables {
  int n_shells, n_orb, n_lab, lmax;
  int mult[8], lab_off[8];
  int shell_l[16], shell_off[17], orb_shell[32];
  int cg_off[4 * 4 * 8];
  const int* kidx;     // [(a * n_shells + b) * 8 + L] -> k
  const int* pair;     // [lab_off-free index: L * 256 + k] -> a * 16 + b
  const float* cg;
};

// Builds the template tables on the host; the device arrays go to `ws` (asynchronous
// copies on `st` from pageable host memory, staged before the call returns).
egnn_status make_tables(const int32_t* shell_l, int32_t n_shells, LabelTables& T, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
  if (!shell_l || n_shells < 1 || n_shells > 16) return EGNN_ERR_INVALID_ARG;
  memset(&T, 0, sizeof(T));
  T.n_shells = n_shells;
  int o = 0, lmax = 0;
  for (int a = 0; a < n_shells; ++a) {
    const int l = shell_l[a];
    if (l < 0 || l > 3) return EGNN_ERR_UNSUPPORTED;
    if (o + 2 * l + 1 > 32) return EGNN_ERR_UNSUPPORTED;
    T.shell_l[a] = l;
    T.shell_off[a] = o;
    for (int i = 0; i < 2 * l + 1; ++i) T.orb_shell[o + i] = a;
    o += 2 * l + 1;
    lmax = 2 * l > lmax ? 2 * l : lmax;
  }
  T.shell_off[n_shells] = o;
  T.n_orb = o;
  T.lmax = lmax;
  std::vector<int> kidx(n_shells * n_shells * 8, 0), pair(8 * 256, 0);
  for (int a = 0; a < n_shells; ++a)
    for (int b = 0; b < n_shells; ++b)
      for (int L = abs(shell_l[a] - shell_l[b]); L <= shell_l[a] + shell_l[b]; ++L) {
        pair[L * 256 + T.mult[L]] = a * 16 + b;
        kidx[(a * n_shells + b) * 8 + L] = T.mult[L]++;
      }
  int lab = 0;
  for (int L = 0; L < 8; ++L) {
    T.lab_off[L] = lab;
    if (L <= lmax) lab += (2 * L + 1) * T.mult[L];
  }
  T.n_lab = lab;
  std::vector<float> cg;
  for (int la = 0; la <= 3; ++la)
    for (int lb = 0; lb <= 3; ++lb)
      for (int L = abs(la - lb); L <= la + lb; ++L) {
        T.cg_off[(la * 4 + lb) * 8 + L] = (int)cg.size();
        real_cg(la, lb, L, cg);
      }
  const size_t b0 = kidx.size() * 4, b1 = (b0 + 15) & ~(size_t)15;
  const size_t b2 = b1 + pair.size() * 4, b3 = (b2 + 15) & ~(size_t)15;
  if (!ws || ws_bytes < b3 + cg.size() * 4) return EGNN_ERR_INVALID_ARG;
  char* w = (char*)ws;
  EGNN_CUDA_TRY(cudaMemcpyAsync(w, kidx.data(), b0, cudaMemcpyHostToDevice, st));
  EGNN_CUDA_TRY(cudaMemcpyAsync(w + b1, pair.data(), pair.size() * 4, cudaMemcpyHostToDevice, st));
  EGNN_CUDA_TRY(cudaMemcpyAsync(w + b3, cg.data(), cg.size() * 4, cudaMemcpyHostToDevice, st));
  T.kidx = (const int*)w;
  T.pair = (const int*)(w + b1);
  T.cg = (const float*)(w + b3);
  return EGNN_OK;
}

// Label -> block: one thread per matrix element of `te` blocks staged per CTA.
__global__ void __launch_bounds__(256) labels_to_blocks_kernel(const float* __restrict__ labels, long long n,
                                                               const __grid_constant__ LabelTables T, int te,
                                                               float* __restrict__ blocks) {
  extern __shared__ float lsm[];   // [te][n_lab]
  const int nlab = T.n_lab, norb = T.n_orb, nb = norb * norb;
  for (long long g0 = (long long)blockIdx.x * te; g0 < n; g0 += (long long)gridDim.x * te) {
    const int ne = (int)min((long long)te, n - g0);
    __syncthreads();
    for (int i = threadIdx.x; i < ne * nlab; i += blockDim.x) lsm[i] = labels[g0 * nlab + i];
    __syncthreads();
    for (int i = threadIdx.x; i < ne * nb; i += blockDim.x) {
      const int e = i / nb, q = i - e * nb;
      const int ri = q / norb, cj = q - ri * norb;
      const int a = T.orb_shell[ri], b = T.orb_shell[cj];
      const int la = T.shell_l[a], lb = T.shell_l[b];
      const int ia = ri - T.shell_off[a], jb = cj - T.shell_off[b];
      float v = 0.f;
      for (int L = abs(la - lb); L <= la + lb; ++L) {
        const int k = T.kidx[(a * T.n_shells + b) * 8 + L], mult = T.mult[L];
        const float* c = T.cg + T.cg_off[(la * 4 + lb) * 8 + L] + (ia * (2 * lb + 1) + jb) * (2 * L + 1);
        const float* h = lsm + e * nlab + T.lab_off[L] + k;
        for (int M = 0; M < 2 * L + 1; ++M) v = fmaf(c[M], h[M * mult], v);
      }
      blocks[(g0 + e) * nb + q] = v;
    }
  }
}

// Block -> label: one thread per label of `te` blocks staged per CTA.
__global__ void __launch_bounds__(256) blocks_to_labels_kernel(const float* __restrict__ blocks, long long n,
                                                               const __grid_constant__ LabelTables T, int te,
                                                               float* __restrict__ labels) {
  extern __shared__ float bsm[];   // [te][n_orb * n_orb]
  const int nlab = T.n_lab, norb = T.n_orb, nb = norb * norb;
  for (long long g0 = (long long)blockIdx.x * te; g0 < n; g0 += (long long)gridDim.x * te) {
    const int ne = (int)min((long long)te, n - g0);
    __syncthreads();
    for (int i = threadIdx.x; i < ne * nb; i += blockDim.x) bsm[i] = blocks[g0 * nb + i];
    __syncthreads();
    for (int i = threadIdx.x; i < ne * nlab; i += blockDim.x) {
      const int e = i / nlab;
      int q = i - e * nlab, L = 0;
      while (q >= (2 * L + 1) * T.mult[L]) {
        q -= (2 * L + 1) * T.mult[L];
        ++L;
      }
      const int mult = T.mult[L], M = q / mult, k = q - M * mult;
      const int ab = T.pair[L * 256 + k], a = ab >> 4, b = ab & 15;
      const int la = T.shell_l[a], lb = T.shell_l[b], na = 2 * la + 1, nbb = 2 * lb + 1;
      const float* c = T.cg + T.cg_off[(la * 4 + lb) * 8 + L] + M;
      const float* h = bsm + e * nb + T.shell_off[a] * norb + T.shell_off[b];
      float v = 0.f;
      for (int ia = 0; ia < na; ++ia)
        for (int jb = 0; jb < nbb; ++jb) v = fmaf(c[(ia * nbb + jb) * (2 * L + 1)], h[ia * norb + jb], v);
      labels[(g0 + e) * nlab + (i - e * nlab)] = v;
    }
  }
}

int pick_te(int per_item_floats, int per_item_work) {
  int te = 1;
  while (te < 64 && (te * 2) * per_item_floats * 4 <= 48 * 1024 && te * per_item_work < 1024) te *= 2;
  return te;
}

// ---- assembly ----
// Row block d: 1 (on-site) + the distinct sources s != d of d's edges (edges sorted by
// source within the segment, so equal sources are adjacent).  One warp per atom.
__global__ void h_count_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ src, int n,
                               int32_t* __restrict__ counts) {
  const int d = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (d >= n) return;
  const int b = row_ptr[d], en = row_ptr[d + 1];
  int c = 0;
  for (int e = b + lane; e < en; e += 32) {
    const int s = src[e];
    c += (s != d && (e == b || src[e - 1] != s)) ? 1 : 0;
  }
  for (int off = 16; off; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
  if (lane == 0) counts[d] = 1 + c;
}

// Exclusive scan of n counts by one CTA; out[n] = total.
__global__ void h_scan_kernel(const int32_t* __restrict__ in, int32_t* __restrict__ out, int n) {
  __shared__ long long part[1024];
  const int t = threadIdx.x, T = blockDim.x;
  const int per = (n + T - 1) / T, b = t * per, e = min(n, b + per);
  long long s = 0;
  for (int i = b; i < e; ++i) s += in[i];
  part[t] = s;
  __syncthreads();
  for (int off = 1; off < T; off <<= 1) {
    const long long v = t >= off ? part[t - off] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  long long run = t == 0 ? 0 : part[t - 1];
  for (int i = b; i < e; ++i) {
    out[i] = (int32_t)run;
    run += in[i];
  }
  if (t == T - 1) out[n] = (int32_t)part[T - 1];
}

// One CTA per row block d: its column list, then each block as the sum of its edges'
// blocks (in edge order) plus, for column d, the on-site block.
__global__ void __launch_bounds__(256) h_fill_kernel(const int32_t* __restrict__ row_ptr,
                                                     const int32_t* __restrict__ src, int n,
                                                     const float* __restrict__ onsite,
                                                     const float* __restrict__ edge_blocks, int nb,
                                                     const int32_t* __restrict__ bsr_row_ptr,
                                                     int32_t* __restrict__ bsr_col, float* __restrict__ bsr_val) {
  __shared__ int run_b[4097], run_s[4096];
  __shared__ int nrun, self_run;
  const int d = blockIdx.x, tid = threadIdx.x;
  const int b = row_ptr[d], en = row_ptr[d + 1];
  if (tid == 0) {
    nrun = 0;
    self_run = -1;
  }
  __syncthreads();
  // runs of equal source, in order (the segment holds at most 4096 edges)
  for (int e0 = b; e0 < en; e0 += blockDim.x) {
    const int e = e0 + tid;
    const bool start = e < en && (e == b || src[e - 1] != src[e]);
    const unsigned bal = __ballot_sync(0xffffffffu, start);
    __shared__ int wbase[8];
    if ((tid & 31) == 0) wbase[tid >> 5] = __popc(bal);
    __syncthreads();
    int k = nrun;
    for (int w = 0; w < (tid >> 5); ++w) k += wbase[w];
    k += __popc(bal & ((1u << (tid & 31)) - 1u));
    if (start) {
      run_b[k] = e;
      run_s[k] = src[e];
    }
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += wbase[w];
      nrun += tot;
    }
    __syncthreads();
  }
  if (tid == 0) {
    run_b[nrun] = en;
    for (int k = 0; k < nrun; ++k)
      if (run_s[k] == d) self_run = k;
  }
  __syncthreads();
  // output block j in column order: runs with s < d, the on-site block (with the run
  // of s == d, if any), runs with s > d
  int n_lo = 0;
  for (int k = 0; k < nrun; ++k) n_lo += run_s[k] < d ? 1 : 0;
  const int row0 = bsr_row_ptr[d], nblk = bsr_row_ptr[d + 1] - row0;
  for (int j = 0; j < nblk; ++j) {
    int k = -1;   // run of block j (-1: on-site only)
    int col = d;
    if (j < n_lo) {
      k = j;
      col = run_s[k];
    } else if (j == n_lo) {
      k = self_run;
    } else {
      k = j - 1 + (self_run >= 0 ? 1 : 0);
      col = run_s[k];
    }
    if (tid == 0) bsr_col[row0 + j] = col;
    float* out = bsr_val + (size_t)(row0 + j) * nb;
    for (int q = tid; q < nb; q += blockDim.x) {
      float v = col == d ? onsite[(size_t)d * nb + q] : 0.f;
      if (k >= 0)
        for (int e = run_b[k]; e < run_b[k + 1]; ++e) v += edge_blocks[(size_t)e * nb + q];
      out[q] = v;
    }
  }
}

}  // namespace

extern "C" int32_t egnn_label_count(const int32_t* shell_l, int32_t n_shells) {
  if (!shell_l || n_shells < 1 || n_shells > 16) return 0;
  int mult[8] = {0}, lmax = 0;
  for (int a = 0; a < n_shells; ++a) {
    if (shell_l[a] < 0 || shell_l[a] > 3) return 0;
    lmax = 2 * shell_l[a] > lmax ? 2 * shell_l[a] : lmax;
    for (int b = 0; b < n_shells; ++b)
      for (int L = abs(shell_l[a] - shell_l[b]); L <= shell_l[a] + shell_l[b]; ++L) ++mult[L];
  }
  int lab = 0;
  for (int L = 0; L <= lmax; ++L) lab += (2 * L + 1) * mult[L];
  return lab;
}

extern "C" egnn_status egnn_labels_to_blocks(const float* labels, int64_t n, const int32_t* shell_l,
                                             int32_t n_shells, float* blocks, void* workspace, size_t ws_bytes,
                                             void* cuda_stream) {
  if (n < 0 || (n > 0 && (!labels || !blocks))) return EGNN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)cuda_stream;
  LabelTables T;
  egnn_status s = make_tables(shell_l, n_shells, T, workspace, ws_bytes, st);
  if (s != EGNN_OK || n == 0) return s;
  const int te = pick_te(T.n_lab, T.n_orb * T.n_orb);
  const long long groups = (n + te - 1) / te;
  const int grid = (int)(groups < 148 * 16 ? groups : 148 * 16);
  labels_to_blocks_kernel<<<grid, 256, (size_t)te * T.n_lab * 4, st>>>(labels, n, T, te, blocks);
  EGNN_CUDA_TRY(cudaGetLastError());
  return EGNN_OK;
}

extern "C" egnn_status egnn_blocks_to_labels(const float* blocks, int64_t n, const int32_t* shell_l,
                                             int32_t n_shells, float* labels, void* workspace, size_t ws_bytes,
                                             void* cuda_stream) {
  if (n < 0 || (n > 0 && (!labels || !blocks))) return EGNN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)cuda_stream;
  LabelTables T;
  egnn_status s = make_tables(shell_l, n_shells, T, workspace, ws_bytes, st);
  if (s != EGNN_OK || n == 0) return s;
  const int te = pick_te(T.n_orb * T.n_orb, T.n_lab);
  const long long groups = (n + te - 1) / te;
  const int grid = (int)(groups < 148 * 16 ? groups : 148 * 16);
  blocks_to_labels_kernel<<<grid, 256, (size_t)te * T.n_orb * T.n_orb * 4, st>>>(blocks, n, T, te, labels);
  EGNN_CUDA_TRY(cudaGetLastError());
  return EGNN_OK;
}

extern "C" egnn_status egnn_assemble_hamiltonian(const egnn_graph* g, const float* onsite,
                                                 const float* edge_blocks, int32_t n_orb, int32_t* bsr_row_ptr,
                                                 int32_t* bsr_col, float* bsr_val, int64_t capacity,
                                                 void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (!g || !g->row_ptr || g->n_atoms < 1 || g->n_edges < 0 || (g->n_edges > 0 && (!g->src || !edge_blocks)))
    return EGNN_ERR_INVALID_ARG;
  if (!onsite || !bsr_row_ptr || !bsr_col || !bsr_val || n_orb < 1 || n_orb > 32) return EGNN_ERR_INVALID_ARG;
  if (capacity < (int64_t)g->n_atoms + g->n_edges) return EGNN_ERR_CAPACITY;
  if (!workspace || ws_bytes < (size_t)g->n_atoms * 4) return EGNN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)cuda_stream;
  const int n = g->n_atoms;
  int32_t* counts = (int32_t*)workspace;
  h_count_kernel<<<(n * 32 + 255) / 256, 256, 0, st>>>(g->row_ptr, g->src, n, counts);
  h_scan_kernel<<<1, 1024, 0, st>>>(counts, bsr_row_ptr, n);
  h_fill_kernel<<<n, 256, 0, st>>>(g->row_ptr, g->src, n, onsite, edge_blocks, n_orb * n_orb, bsr_row_ptr, bsr_col,
                                   bsr_val);
  EGNN_CUDA_TRY(cudaGetLastError());
  return EGNN_OK;
}
