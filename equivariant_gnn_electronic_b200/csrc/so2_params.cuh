// Launch parameters shared by the eSCN layer / head kernels (CUDA path only).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

struct So2Params {
  int n_atoms;
  long long n_edges;
  int lmax, mmax, C, H, K, L, L2, nrows, wfl, te, dtype;
  float rcut;
  const int32_t* row_ptr;
  const int32_t* src;
  const float* dist;
  const float* wig;
  const void* node_in;
  void* node_out;
  float* blocks;
  int32_t* status;
  int woff[8];     // Wigner float offset of degree l inside an edge's record
  int row0[8];     // kept-row index of (l, m = 0)
  int row_l[32];   // degree of each kept row
  int row_m[32];   // order of each kept row
  int coef_l[64];  // degree of each coefficient index l*l + l + m
};

struct So2Weights {
  const void *W1, *b1, *W2, *b2, *W0;
  const void* Wm[2][2];   // [m-1][0] = W_m1, [m-1][1] = W_m2
  const void *A, *bA;
  const void* U[8];
};

struct HeadTables {
  int n_orb, n_lab, n_shells;
  int lab_off[8];     // label offset of degree L (labels ordered L, then M, then k)
  int mult[8];        // shell pairs containing L
  int shell_l[16];
  int shell_off[17];
  int orb_shell[32];
  int cg_off[4 * 4 * 8];  // offset of C^{L}(la, lb) in cg, index (la*4 + lb)*8 + L
  const int* kidx;        // [(a*n_shells + b)*8 + L] -> label multiplicity index k
  const float* cg;        // real Clebsch-Gordan matrices, row-major [(2la+1)(2lb+1)][2L+1]
};

size_t so2_simt_smem_bytes(const So2Params& P, int te);
int so2_simt_pick_te(const So2Params& P, int head_labels);
cudaError_t launch_layer_simt(So2Params P, So2Weights W, cudaStream_t st);
cudaError_t launch_head_simt(So2Params P, So2Weights W, HeadTables T, cudaStream_t st);

// Real Clebsch-Gordan matrix C^L(la, lb) of the basis of egnn.h, row-major
// [(2la+1)(2lb+1)][2L+1], appended to `out` (api.cu).
void real_cg(int la, int lb, int L, std::vector<float>& out);
