// Host side of the C ABI declared in include/egnn.h: argument checks, parameter
// packing, Clebsch-Gordan tables, dispatch to the kernels.
#include <math.h>
#include <string.h>

#include <complex>
#include <vector>

#include "common.cuh"
#include "so2_params.cuh"
#include "so2_tc.cuh"

size_t egnn_graph_workspace_bytes(int32_t n_atoms);   // graph.cu

namespace {

size_t dtype_size(int dt) { return dt == EGNN_BF16 ? 2 : 4; }

egnn_status check_desc(const egnn_layer_desc* d) {
  if (!d) return EGNN_ERR_INVALID_ARG;
  if (d->dtype != EGNN_FP32 && d->dtype != EGNN_BF16) return EGNN_ERR_UNSUPPORTED;
  if (d->lmax < 0 || d->lmax > 6 || d->mmax < 0 || d->mmax > 2 || d->mmax > d->lmax) return EGNN_ERR_UNSUPPORTED;
  if (d->channels < 1 || d->channels > 128 || d->heads < 1 || d->heads > 16) return EGNN_ERR_UNSUPPORTED;
  if (d->channels % d->heads) return EGNN_ERR_UNSUPPORTED;
  if (d->n_rbf < 2 || d->n_rbf > 64) return EGNN_ERR_UNSUPPORTED;
  if (!(d->rcut > 0.f)) return EGNN_ERR_INVALID_ARG;
  return EGNN_OK;
}

egnn_status check_graph(const egnn_graph* g, const egnn_layer_desc* d) {
  if (!g || !g->row_ptr || !g->status || g->n_atoms < 1) return EGNN_ERR_INVALID_ARG;
  if (g->n_edges < 0 || g->n_edges > g->capacity) return EGNN_ERR_INVALID_ARG;
  if (g->n_edges > 0 && (!g->src || !g->dist || !g->wigner)) return EGNN_ERR_INVALID_ARG;
  if (g->lmax != d->lmax || g->mmax != d->mmax) return EGNN_ERR_INVALID_ARG;
  return EGNN_OK;
}

void fill_params(So2Params& P, const egnn_graph* g, const egnn_layer_desc* d) {
  memset(&P, 0, sizeof(P));
  P.n_atoms = g->n_atoms;
  P.n_edges = g->n_edges;
  P.lmax = d->lmax;
  P.mmax = d->mmax;
  P.C = d->channels;
  P.H = d->heads;
  P.K = d->n_rbf;
  P.L = d->lmax + 1;
  P.L2 = P.L * P.L;
  P.wfl = egnn_wigner_floats(d->lmax, d->mmax);
  P.dtype = d->dtype;
  P.rcut = d->rcut;
  P.row_ptr = g->row_ptr;
  P.src = g->src;
  P.dist = g->dist;
  P.wig = g->wigner;
  P.status = g->status;
  int r = 0;
  for (int l = 0; l <= d->lmax; ++l) {
    int ml = l < d->mmax ? l : d->mmax;
    P.woff[l] = egnn_wig_off(l, d->mmax);
    P.row0[l] = r + ml;
    for (int m = -ml; m <= ml; ++m) {
      P.row_l[r] = l;
      P.row_m[r] = m;
      ++r;
    }
    for (int m = -l; m <= l; ++m) P.coef_l[l * l + l + m] = l;
  }
  P.nrows = r;
}

// Carves the packed weight buffer (order documented in egnn.h); returns elements used.
size_t carve_so2(So2Weights& W, const char* base, const egnn_layer_desc* d, bool attention) {
  const size_t es = dtype_size(d->dtype);
  const size_t L = d->lmax + 1, C = d->channels, K = d->n_rbf;
  size_t o = 0;
  auto take = [&](size_t n) { const void* p = base + o * es; o += n; return p; };
  memset(&W, 0, sizeof(W));
  W.W1 = take(C * K);
  W.b1 = take(C);
  W.W2 = take(L * 2 * C * C);
  W.b2 = take(L * 2 * C);
  W.W0 = take(L * C * L * 2 * C);
  for (int m = 1; m <= d->mmax; ++m) {
    size_t nm = L - m;
    W.Wm[m - 1][0] = take(nm * C * nm * 2 * C);
    W.Wm[m - 1][1] = take(nm * C * nm * 2 * C);
  }
  if (attention) {
    W.A = take(d->heads * L * C);
    W.bA = take(d->heads);
  }
  return o;
}

// ---------------- tensor-core layer plan ----------------
bool tc_eligible(const egnn_layer_desc* d) {
  return d->dtype == EGNN_BF16 && d->channels == 128 && d->lmax >= 1 && d->lmax <= 6 && d->mmax <= 2 &&
         d->heads <= 16 && 128 % d->heads == 0;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Pass list: radial-gate passes (256 columns each), then the SO(2) blocks
// |m| = 0..mmax, each block's output rows split into accumulators of at most
// kTcAccCols TMEM columns.  With `mult`
// (head, label mode) the output rows of block b are the labels (l >= b, k < mult_l)
// instead of the channels (l >= b, c < C).  Returns false if the plan needs more
// passes than TcParams holds.
bool tc_plan(const egnn_layer_desc* d, TcParams& P, const int* mult = nullptr) {
  const int L = d->lmax + 1, C = d->channels;
  const bool label = mult != nullptr;
  P.npass = 0;
  P.label_mode = label ? 1 : 0;
  long long boff = 0;
  int roff = 0;
  auto add = [&](int kind, int block, int ntot, int nk) -> bool {
    const int step = kind == 0 ? 256 : kTcAccCols;   // gate passes alternate two 256-column accumulators
    for (int off = 0; off < ntot; off += step) {
      if (P.npass >= 32) return false;
      TcPass& q = P.pass[P.npass++];
      q.kind = kind;
      q.block = block;
      q.n = ntot - off < step ? ntot - off : step;
      q.n_off = off;
      q.nk = nk;
      q.last_of_kind = 0;
      q.np = 0;
      q.boff = boff;
      q.roff = kind == 1 ? roff : 0;
      if (kind == 1) roff += q.n;
      boff += (long long)q.n * nk * 128;
    }
    P.pass[P.npass - 1].last_of_kind = 1;
    return true;
  };
  if (!add(0, 0, L * 2 * C, C / 64)) return false;
  int ycol = 0;
  P.ybase[0] = ycol;
  int nr0 = L * C;
  if (label) {
    nr0 = 0;
    for (int l = 0; l < L; ++l) nr0 += mult[l];
    P.hnr[0] = nr0;
    P.hroff[0] = roff;
    nr0 = (nr0 + 31) & ~31;
  }
  if (!add(1, 0, nr0, L * 2 * C / 64)) return false;
  ycol += L * C;
  for (int b = 1; b <= d->mmax; ++b) {
    // rows [o0, o0 + np) of y+ and of y-: B = [W_b1 rows ; W_b2 rows] for those outputs,
    // K = the (l, channel) index shared by x+ and x- (each K block feeds 4 MMAs)
    int nC = (L - b) * C;
    if (label) {
      nC = 0;
      for (int l = b; l < L; ++l) nC += mult[l];
      P.hnr[b] = nC;
      P.hroff[b] = roff;
    }
    const int kblocks = (L - b) * 2 * C / 64;
    P.ybase[b] = ycol;
    ycol += 2 * (L - b) * C;
    for (int o0 = 0; o0 < nC; o0 += kTcPairRows) {
      if (P.npass >= 32) return false;
      TcPass& q = P.pass[P.npass++];
      q.kind = 1;
      q.block = b;
      q.np = nC - o0 < kTcPairRows ? nC - o0 : kTcPairRows;
      if (label) q.np = (q.np + 15) & ~15;
      q.n = 2 * q.np;
      q.n_off = o0;
      q.nk = kblocks;
      q.last_of_kind = 0;
      q.boff = boff;
      q.roff = roff;
      roff += q.n;
      boff += (long long)q.n * kblocks * 128;
    }
  }
  // A tiles of one edge tile (gate_rotate output): block 0 one per (l, 64 channels),
  // |m| = b > 0 an x+ / x- pair per (l >= b, 64 channels)
  const int kpl = 2 * C / 64;
  P.xbase[0] = 0;
  P.nch = L * kpl;
  for (int b = 1; b <= d->mmax; ++b) {
    P.xbase[b] = P.nch;
    P.nch += 2 * (L - b) * kpl;
  }
  P.ncols_y = ycol;
  P.y0_bytes = L * C * 4;
  P.y_row_bytes = label ? roff * 4 : P.y0_bytes + (ycol - L * C) * 2;
  P.gcols = L * 2 * C;
  P.wprep_bytes = boff;
  if (label)
    for (int l = 0; l < 8; ++l) P.mult[l] = l < L ? mult[l] : 0;
  return true;
}

struct TcWorkspace {
  size_t wprep, x, y, total;
};

TcWorkspace tc_workspace(const egnn_layer_desc* d, int64_t n_edges, int32_t n_atoms) {
  TcParams P;
  memset(&P, 0, sizeof(P));
  tc_plan(d, P);
  TcWorkspace w;
  size_t E = n_edges > 0 ? (size_t)n_edges : 0;
  const size_t tch = (size_t)tc_chunk_tiles((int)((E + 127) / 128));
  w.wprep = 0;
  w.x = align_up((size_t)P.wprep_bytes, 1024);
  w.y = w.x + align_up(tch * P.nch * 16384, 1024);
  (void)n_atoms;
  w.total = w.y + align_up(E * (size_t)P.y_row_bytes, 1024) + 1024;
  return w;
}

// Workspace of the fused tensor-core layer: prepared weights, the A tiles of one range
// of edge tiles, the per-CTA y0 stash, per-atom accumulators and two
// partial records per edge tile.  Nothing in it is stored per edge except the
// records (2 (L^2 C + 32) floats per 128 edges).
struct LayerWorkspace {
  size_t wprep, x, stash, edst, acc, slots, total;
  int rec_floats;
};

LayerWorkspace layer_workspace(const egnn_layer_desc* d, int64_t n_edges, int32_t n_atoms) {
  TcParams P;
  memset(&P, 0, sizeof(P));
  tc_plan(d, P);
  LayerWorkspace w;
  const size_t E = n_edges > 0 ? (size_t)n_edges : 0, N = n_atoms > 0 ? (size_t)n_atoms : 0;
  const size_t L = d->lmax + 1, C = d->channels;
  const size_t n_tiles = (E + 127) / 128;
  const size_t tch = (size_t)tc_chunk_tiles((int)n_tiles);
  w.rec_floats = (int)(L * L * C + 32);
  w.wprep = 0;
  w.x = align_up((size_t)P.wprep_bytes, 1024);
  w.stash = w.x + align_up(tch * P.nch * 16384, 1024);
  w.edst = w.stash + align_up((size_t)kTcMaxGrid * L * 128 * C * 2, 1024);
  w.acc = w.edst + align_up(E * 4, 1024);
  w.slots = w.acc + align_up(N * L * L * C * 4, 1024);
  w.total = w.slots + align_up(n_tiles * 2 * (size_t)w.rec_floats * 4, 1024) + 1024;
  return w;
}

// Fills the tensor-core launch parameters for graph g, weights W and a 1024-aligned
// workspace (label mode with `mult`; the fused layer's layout with `layer`); returns
// false if the pass plan does not fit.
bool fill_tc(TcParams& T, TcWeights& TW, const egnn_graph* g, const egnn_layer_desc* desc, const So2Weights& W,
             const void* node_in, void* node_out, uint8_t* ws, const int* mult = nullptr,
             bool layer = false) {
  TcWorkspace wl = tc_workspace(desc, g->n_edges, g->n_atoms);
  memset(&T, 0, sizeof(T));
  if (!tc_plan(desc, T, mult)) return false;
  T.n_atoms = g->n_atoms;
  T.n_edges = g->n_edges;
  T.n_tiles = (int)((g->n_edges + 127) / 128);
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  T.grid = nsm < kTcMaxGrid ? nsm : kTcMaxGrid;
  if (T.grid > T.n_tiles) T.grid = T.n_tiles > 0 ? T.n_tiles : 1;
  T.lmax = desc->lmax;
  T.mmax = desc->mmax;
  T.C = desc->channels;
  T.H = desc->heads;
  T.K = desc->n_rbf;
  T.L = desc->lmax + 1;
  T.L2 = T.L * T.L;
  T.wfl = egnn_wigner_floats(desc->lmax, desc->mmax);
  T.rcut = desc->rcut;
  T.row_ptr = g->row_ptr;
  T.src = g->src;
  T.dist = g->dist;
  T.wig = g->wigner;
  T.status = g->status;
  T.node_in = (const __nv_bfloat16*)node_in;
  T.node_out = (__nv_bfloat16*)node_out;
  for (int l = 0; l <= desc->lmax; ++l) T.woff[l] = egnn_wig_off(l, desc->mmax);
  T.W1 = (const __nv_bfloat16*)W.W1;
  T.b1 = (const __nv_bfloat16*)W.b1;
  T.b2 = (const __nv_bfloat16*)W.b2;
  T.A = (const __nv_bfloat16*)W.A;
  T.bA = (const __nv_bfloat16*)W.bA;
  if (layer) {
    const LayerWorkspace lw = layer_workspace(desc, g->n_edges, g->n_atoms);
    T.wprep = ws + lw.wprep;
    T.X = ws + lw.x;
    T.stash = (__nv_bfloat16*)(ws + lw.stash);
    T.edge_dst = (int32_t*)(ws + lw.edst);
    T.acc_g = (float*)(ws + lw.acc);
    T.slots = (float*)(ws + lw.slots);
    T.rec_floats = lw.rec_floats;
    // Degrees of the fused kernel's two epilogue groups, balanced by rotate-back work
    // ((2l + 1) per kept row: one m = 0 row and two per 0 < b <= min(l, mmax)); group 0
    // starts with a share for the attention logits it also forms.
    double work[8] = {0}, total = 0;
    for (int l = 0; l <= desc->lmax; ++l) {
      const int ml = l < desc->mmax ? l : desc->mmax;
      work[l] = (2.0 * l + 1) * (1 + 2 * ml);
      total += work[l];
    }
    double load[2] = {0.15 * total, 0.0};
    bool done[8] = {false};
    T.own_b = 0;
    for (int it = 0; it <= desc->lmax; ++it) {
      int best = -1;
      for (int l = 0; l <= desc->lmax; ++l)
        if (!done[l] && (best < 0 || work[l] > work[best])) best = l;
      done[best] = true;
      const int gsel = load[1] < load[0] ? 1 : 0;
      load[gsel] += work[best];
      if (gsel) T.own_b |= 1 << best;
    }
  } else {
    T.wprep = ws + wl.wprep;
    T.X = ws + wl.x;
    T.Y = ws + wl.y;
  }
  TW.W2 = (const __nv_bfloat16*)W.W2;
  TW.W0 = (const __nv_bfloat16*)W.W0;
  for (int m = 0; m < 2; ++m)
    for (int k = 0; k < 2; ++k) TW.Wm[m][k] = (const __nv_bfloat16*)W.Wm[m][k];
  return true;
}

uint8_t* align1024(void* p) { return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023); }

}  // namespace

// ---------------- Clebsch-Gordan tables (library side) ----------------
// Complex coefficients <j1 m1 j2 m2 | J M> by Racah's closed formula, then the
// unitary change to the real basis of egnn.h (real_m = sum_mu U[m][mu] Y^mu,
// Y^mu with the Condon-Shortley phase):  C_real = (U_la (x) U_lb) C U_L^dagger.
// The result is real up to one global phase, removed before the sign rule
// (first non-zero entry of column M = -L positive).
namespace {

double fact(int n) {
  double r = 1;
  for (int i = 2; i <= n; ++i) r *= i;
  return r;
}

double cg_complex(int j1, int m1, int j2, int m2, int J, int M) {
  if (m1 + m2 != M || abs(m1) > j1 || abs(m2) > j2 || abs(M) > J) return 0.0;
  double pre = sqrt((2 * J + 1) * fact(J + j1 - j2) * fact(J - j1 + j2) * fact(j1 + j2 - J) /
                    fact(j1 + j2 + J + 1));
  pre *= sqrt(fact(J + M) * fact(J - M) * fact(j1 - m1) * fact(j1 + m1) * fact(j2 - m2) * fact(j2 + m2));
  double s = 0.0;
  for (int k = 0; k <= j1 + j2 + J; ++k) {
    int a[6] = {k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k};
    bool ok = true;
    double den = 1.0;
    for (int t = 0; t < 6; ++t) {
      if (a[t] < 0) ok = false;
      else den *= fact(a[t]);
    }
    if (ok) s += ((k & 1) ? -1.0 : 1.0) / den;
  }
  return pre * s;
}

std::complex<double> real_from_complex(int m, int mu) {
  const double r = 1.0 / sqrt(2.0);
  if (m == 0) return mu == 0 ? 1.0 : 0.0;
  if (m > 0) {
    if (mu == m) return ((m & 1) ? -r : r);
    if (mu == -m) return r;
    return 0.0;
  }
  int am = -m;
  if (mu == am) return std::complex<double>(0.0, (am & 1) ? r : -r);
  if (mu == -am) return std::complex<double>(0.0, r);
  return 0.0;
}

}  // namespace

// Real Clebsch-Gordan matrix C^L(la, lb), row-major [(2la+1)(2lb+1)][2L+1], appended to out.
void real_cg(int la, int lb, int L, std::vector<float>& out) {
  int na = 2 * la + 1, nb = 2 * lb + 1, nl = 2 * L + 1;
  std::vector<std::complex<double>> C(na * nb * nl);
  for (int ma = -la; ma <= la; ++ma)
    for (int mb = -lb; mb <= lb; ++mb)
      for (int m = -L; m <= L; ++m) {
        std::complex<double> s = 0.0;
        for (int ua = -la; ua <= la; ++ua) {
          std::complex<double> fa = real_from_complex(ma, ua);
          if (fa == 0.0) continue;
          for (int ub = -lb; ub <= lb; ++ub) {
            std::complex<double> fb = real_from_complex(mb, ub);
            if (fb == 0.0 || abs(ua + ub) > L) continue;
            s += fa * fb * cg_complex(la, ua, lb, ub, L, ua + ub) * std::conj(real_from_complex(m, ua + ub));
          }
        }
        C[((ma + la) * nb + (mb + lb)) * nl + (m + L)] = s;
      }
  double nr = 0, ni = 0;
  for (auto& c : C) {
    nr += c.real() * c.real();
    ni += c.imag() * c.imag();
  }
  std::vector<double> R(C.size());
  for (size_t i = 0; i < C.size(); ++i) R[i] = nr >= ni ? C[i].real() : C[i].imag();
  for (int r = 0; r < na * nb; ++r) {
    double v = R[(size_t)r * nl];
    if (fabs(v) > 1e-9) {
      if (v < 0)
        for (auto& x : R) x = -x;
      break;
    }
  }
  for (double x : R) out.push_back((float)x);
}


extern "C" size_t egnn_workspace_bytes(int32_t which, const egnn_layer_desc* desc, int32_t n_atoms,
                                       int64_t n_edges) {
  (void)n_edges;
  switch (which) {
    case EGNN_WS_BUILD_GRAPH:
      return egnn_graph_workspace_bytes(n_atoms);
    case EGNN_WS_LAYER:
      if (desc && check_desc(desc) == EGNN_OK && tc_eligible(desc))
        return layer_workspace(desc, n_edges, n_atoms).total;
      return 256;
    case EGNN_WS_LABELS:
      return 1024 * 1024;
    case EGNN_WS_ASSEMBLY:
      return (size_t)(n_atoms > 0 ? n_atoms : 0) * 4 + 256;
    case EGNN_WS_HAMILTONIAN:
      if (desc && check_desc(desc) == EGNN_OK && tc_eligible(desc))
        return tc_workspace(desc, n_edges, n_atoms).total + 1024 * 1024;
      return 64 * 1024;
    default:
      return 0;
  }
  (void)desc;
}

extern "C" egnn_status egnn_layer_forward(const egnn_graph* g, const egnn_layer_desc* desc,
                                          const void* weights, const void* node_in, void* node_out,
                                          void* workspace, size_t ws_bytes, void* cuda_stream) {
  egnn_status s = check_desc(desc);
  if (s != EGNN_OK) return s;
  if ((s = check_graph(g, desc)) != EGNN_OK) return s;
  if (!weights || !node_in || !node_out) return EGNN_ERR_INVALID_ARG;
  {
    // the aggregation reads neighbours' rows of node_in while other CTAs write node_out:
    // the two byte ranges must be disjoint
    const size_t bytes = (size_t)g->n_atoms * (desc->lmax + 1) * (desc->lmax + 1) * desc->channels *
                         dtype_size(desc->dtype);
    const uintptr_t a = (uintptr_t)node_in, b = (uintptr_t)node_out;
    if (a < b + bytes && b < a + bytes) return EGNN_ERR_INVALID_ARG;
  }
  cudaStream_t st = (cudaStream_t)cuda_stream;
  if (tc_eligible(desc)) {
    const LayerWorkspace wl = layer_workspace(desc, g->n_edges, g->n_atoms);
    if (!workspace || ws_bytes < wl.total) return EGNN_ERR_INVALID_ARG;
    if (((uintptr_t)weights | (uintptr_t)node_in | (uintptr_t)node_out) & 15) return EGNN_ERR_INVALID_ARG;
    uint8_t* ws = align1024(workspace);
    So2Weights W;
    carve_so2(W, (const char*)weights, desc, true);
    TcParams T;
    TcWeights TW;
    fill_tc(T, TW, g, desc, W, node_in, node_out, ws, nullptr, true);
    EGNN_CUDA_TRY(launch_layer_fused(T, TW, st));
    return EGNN_OK;
  }
  So2Params P;
  fill_params(P, g, desc);
  P.node_in = node_in;
  P.node_out = node_out;
  So2Weights W;
  carve_so2(W, (const char*)weights, desc, true);
  P.te = so2_simt_pick_te(P, 0);
  if (P.te < 1) return EGNN_ERR_UNSUPPORTED;
  EGNN_CUDA_TRY(launch_layer_simt(P, W, st));
  return EGNN_OK;
}

extern "C" egnn_status egnn_hamiltonian_blocks(const egnn_graph* g, const egnn_layer_desc* desc,
                                               const void* head_weights, const int32_t* shell_l,
                                               int32_t n_shells, const void* node_emb, float* blocks,
                                               void* workspace, size_t ws_bytes, void* cuda_stream) {
  egnn_status s = check_desc(desc);
  if (s != EGNN_OK) return s;
  if ((s = check_graph(g, desc)) != EGNN_OK) return s;
  if (!head_weights || !shell_l || !node_emb || (!blocks && g->n_edges > 0)) return EGNN_ERR_INVALID_ARG;
  if (n_shells < 1 || n_shells > 16) return EGNN_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < egnn_workspace_bytes(EGNN_WS_HAMILTONIAN, desc, g->n_atoms, g->n_edges))
    return EGNN_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)cuda_stream;
  HeadTables T;
  memset(&T, 0, sizeof(T));
  T.n_shells = n_shells;
  int o = 0;
  for (int a = 0; a < n_shells; ++a) {
    int l = shell_l[a];
    if (l < 0 || l > 3) return EGNN_ERR_UNSUPPORTED;
    T.shell_l[a] = l;
    T.shell_off[a] = o;
    if (o + 2 * l + 1 > 32) return EGNN_ERR_UNSUPPORTED;
    for (int i = 0; i < 2 * l + 1; ++i) T.orb_shell[o + i] = a;
    o += 2 * l + 1;
    for (int b = 0; b < a; ++b)
      if (shell_l[b] + l > desc->lmax) return EGNN_ERR_UNSUPPORTED;
    if (2 * l > desc->lmax) return EGNN_ERR_UNSUPPORTED;
  }
  T.shell_off[n_shells] = o;
  T.n_orb = o;
  // label multiplicities and k index per (a, b, L): pairs lexicographic, a outer
  std::vector<int> kidx(n_shells * n_shells * 8, 0);
  int mult[8] = {0};
  for (int a = 0; a < n_shells; ++a)
    for (int b = 0; b < n_shells; ++b)
      for (int Lc = abs(shell_l[a] - shell_l[b]); Lc <= shell_l[a] + shell_l[b]; ++Lc)
        kidx[(a * n_shells + b) * 8 + Lc] = mult[Lc]++;
  int lab = 0;
  for (int Lc = 0; Lc <= desc->lmax; ++Lc) {
    T.mult[Lc] = mult[Lc];
    T.lab_off[Lc] = lab;
    lab += (2 * Lc + 1) * mult[Lc];
  }
  for (int Lc = desc->lmax + 1; Lc < 8; ++Lc) T.lab_off[Lc] = lab;
  T.n_lab = lab;
  std::vector<float> cg;
  for (int la = 0; la <= 3; ++la)
    for (int lb = 0; lb <= 3; ++lb)
      for (int Lc = abs(la - lb); Lc <= la + lb; ++Lc) {
        T.cg_off[(la * 4 + lb) * 8 + Lc] = (int)cg.size();
        real_cg(la, lb, Lc, cg);
      }
  const bool use_tc = tc_eligible(desc);
  const size_t tc_bytes = use_tc ? tc_workspace(desc, g->n_edges, g->n_atoms).total : 0;
  size_t need = tc_bytes + kidx.size() * sizeof(int) + cg.size() * sizeof(float) + 64;
  if (ws_bytes < need) return EGNN_ERR_INVALID_ARG;
  uint8_t* ws_tc = align1024(workspace);
  char* wsp = use_tc ? (char*)(ws_tc + tc_bytes - 1024) : (char*)workspace;
  EGNN_CUDA_TRY(cudaMemcpyAsync(wsp, kidx.data(), kidx.size() * sizeof(int), cudaMemcpyHostToDevice, st));
  size_t off = (kidx.size() * sizeof(int) + 15) & ~(size_t)15;
  EGNN_CUDA_TRY(cudaMemcpyAsync(wsp + off, cg.data(), cg.size() * sizeof(float), cudaMemcpyHostToDevice, st));
  T.kidx = (const int*)wsp;
  T.cg = (const float*)(wsp + off);

  So2Weights W;
  size_t used = carve_so2(W, (const char*)head_weights, desc, false);
  const size_t es = dtype_size(desc->dtype);
  for (int Lc = 0; Lc <= desc->lmax; ++Lc) {
    if (mult[Lc]) {
      W.U[Lc] = (const char*)head_weights + used * es;
      used += (size_t)mult[Lc] * desc->channels;
    }
  }
  if (use_tc) {
    if (g->n_edges == 0) return EGNN_OK;
    if (((uintptr_t)head_weights | (uintptr_t)node_emb) & 15) return EGNN_ERR_INVALID_ARG;
    // Label mode (U^L folded into the SO(2) weights) when its pass plan fits and its
    // per-edge record is no larger than the channel-space record the workspace holds.
    TcParams TP, probe;
    memset(&probe, 0, sizeof(probe));
    tc_plan(desc, probe);
    const int y_bytes = probe.y_row_bytes;
    memset(&probe, 0, sizeof(probe));
    const bool label = tc_plan(desc, probe, mult) && probe.y_row_bytes <= y_bytes;
    TcWeights TW;
    if (!fill_tc(TP, TW, g, desc, W, node_emb, nullptr, ws_tc, label ? mult : nullptr))
      return EGNN_ERR_UNSUPPORTED;
    for (int Lc = 0; Lc < 8; ++Lc) TP.U[Lc] = (const __nv_bfloat16*)W.U[Lc];
    HeadUPtrs Up;
    for (int Lc = 0; Lc < 8; ++Lc) Up.U[Lc] = (const __nv_bfloat16*)W.U[Lc];
    if (head_tc_smem_bytes(TP, T.n_lab, 1) > 200 * 1024) return EGNN_ERR_UNSUPPORTED;
    HeadLabelTabs LT;
    memset(&LT, 0, sizeof(LT));
    if (label) {
      // label q: its rotate-back terms (Wigner offset, record offset); block entry q: its
      // (label, Clebsch-Gordan coefficient) terms
      const int norb = T.n_orb, nb = norb * norb, R = kTcPairRows;
      std::vector<int> lab((size_t)T.n_lab * 11, 0), tptr(nb + 1, 0);
      std::vector<int2> terms;
      int lb[3][8];
      for (int b = 0; b < 3; ++b) {
        int acc = 0;
        for (int l = 0; l < 8; ++l) {
          lb[b][l] = acc;
          if (l >= b && l <= desc->lmax) acc += mult[l];
        }
      }
      for (int q0 = 0; q0 < T.n_lab; ++q0) {
        int q = q0, Lq = 0;
        while (q >= (2 * Lq + 1) * mult[Lq]) q -= (2 * Lq + 1) * mult[Lq++];
        const int M = q / mult[Lq], k = q - M * mult[Lq];
        const int ml = Lq < desc->mmax ? Lq : desc->mmax, dl = 2 * Lq + 1, D = TP.woff[Lq] + M;
        int* o = &lab[(size_t)q0 * 11];
        o[0] = 2 * ml + 1;
        o[1] = D + ml * dl;
        o[6] = TP.hroff[0] + lb[0][Lq] + k;
        int j = 1;
        for (int b = 1; b <= ml; ++b) {
          const int r = lb[b][Lq] + k, qq = r / R, w = r - qq * R, rest = TP.hnr[b] - R * qq;
          const int npq = rest >= R ? R : ((rest + 15) & ~15), base = TP.hroff[b] + 2 * R * qq + w;
          o[1 + j] = D + (ml + b) * dl;
          o[6 + j++] = base;
          o[1 + j] = D + (ml - b) * dl;
          o[6 + j++] = base + npq;
        }
      }
      for (int q = 0; q < nb; ++q) {
        const int ri = q / norb, cj = q - ri * norb, a = T.orb_shell[ri], b = T.orb_shell[cj];
        const int la = T.shell_l[a], lbb = T.shell_l[b], ia = ri - T.shell_off[a], jb = cj - T.shell_off[b];
        for (int Lc = abs(la - lbb); Lc <= la + lbb; ++Lc) {
          const int k = kidx[(a * n_shells + b) * 8 + Lc];
          const float* cgm = cg.data() + T.cg_off[(la * 4 + lbb) * 8 + Lc] + (ia * (2 * lbb + 1) + jb) * (2 * Lc + 1);
          for (int M = 0; M < 2 * Lc + 1; ++M) {
            int2 tm;
            tm.x = T.lab_off[Lc] + M * mult[Lc] + k;
            memcpy(&tm.y, &cgm[M], 4);
            terms.push_back(tm);
          }
        }
        tptr[q + 1] = (int)terms.size();
      }
      const size_t o_lab = (off + cg.size() * sizeof(float) + 15) & ~(size_t)15;
      const size_t o_ptr = (o_lab + lab.size() * 4 + 15) & ~(size_t)15;
      const size_t o_term = (o_ptr + tptr.size() * 4 + 15) & ~(size_t)15;
      if ((size_t)(wsp - (char*)workspace) + o_term + terms.size() * 8 > ws_bytes) return EGNN_ERR_INVALID_ARG;
      EGNN_CUDA_TRY(cudaMemcpyAsync(wsp + o_lab, lab.data(), lab.size() * 4, cudaMemcpyHostToDevice, st));
      EGNN_CUDA_TRY(cudaMemcpyAsync(wsp + o_ptr, tptr.data(), tptr.size() * 4, cudaMemcpyHostToDevice, st));
      EGNN_CUDA_TRY(cudaMemcpyAsync(wsp + o_term, terms.data(), terms.size() * 8, cudaMemcpyHostToDevice, st));
      LT.n_lab = T.n_lab;
      LT.n_orb = norb;
      LT.n_term = (int)terms.size();
      LT.lab = (const int*)(wsp + o_lab);
      LT.term_ptr = (const int*)(wsp + o_ptr);
      LT.term = (const int2*)(wsp + o_term);
    }
    EGNN_CUDA_TRY(launch_head_tc(TP, TW, T, Up, LT, blocks, st));
    return EGNN_OK;
  }
  So2Params P;
  fill_params(P, g, desc);
  if (2 * P.nrows < P.L2) return EGNN_ERR_UNSUPPORTED;
  P.node_in = node_emb;
  P.blocks = blocks;
  P.te = so2_simt_pick_te(P, T.n_lab);
  if (P.te < 1) return EGNN_ERR_UNSUPPORTED;
  if (g->n_edges == 0) return EGNN_OK;
  EGNN_CUDA_TRY(launch_head_simt(P, W, T, st));
  // the tables live in `workspace`: keep them until the kernel has read them
  return EGNN_OK;
}

extern "C" egnn_status egnn_check_bounded_wait(egnn_graph* g, uint32_t limit_us, void* cuda_stream) {
  if (!g || !g->status || limit_us == 0 || limit_us > 2000000u) return EGNN_ERR_INVALID_ARG;
  EGNN_CUDA_TRY(launch_wait_check(g->status, 1000ull * limit_us, (cudaStream_t)cuda_stream));
  return EGNN_OK;
}

extern "C" egnn_status egnn_profile(int32_t enable) {
  tc_profile_enable(enable != 0);
  return EGNN_OK;
}

extern "C" egnn_status egnn_profile_read(double* gemm_ms, int64_t* launches, int64_t* edges) {
  if (!gemm_ms || !launches || !edges) return EGNN_ERR_INVALID_ARG;
  long long n = 0, e = 0;
  EGNN_CUDA_TRY(tc_profile_read(gemm_ms, &n, &e));
  *launches = n;
  *edges = e;
  return EGNN_OK;
}

extern "C" egnn_status egnn_read_status(const egnn_graph* g, int32_t* code, void* cuda_stream) {
  if (!g || !g->status) return EGNN_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaStream_t st = (cudaStream_t)cuda_stream;
  EGNN_CUDA_TRY(cudaMemcpyAsync(&v, g->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  EGNN_CUDA_TRY(cudaStreamSynchronize(st));
  if (code) *code = v;
  return v ? EGNN_ERR_DEVICE_CHECK : EGNN_OK;
}

extern "C" const char* egnn_status_string(egnn_status s) {
  switch (s) {
    case EGNN_OK: return "ok";
    case EGNN_ERR_INVALID_ARG: return "invalid argument";
    case EGNN_ERR_CAPACITY: return "graph capacity too small (n_edges holds the required count)";
    case EGNN_ERR_UNSUPPORTED: return "unsupported size, dtype or template";
    case EGNN_ERR_CUDA: return "CUDA runtime error";
    case EGNN_ERR_DEVICE_CHECK: return "device-side check failed (see status word)";
  }
  return "unknown status";
}
