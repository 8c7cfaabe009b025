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
//   apply_terms       both directions: groups of blocks (or label vectors) brought into
//                     shared memory by 1-D bulk copies, the next group's copy in flight
//                     while the current one is summed; one output element over a run
//                     of items per work slot, summing its precomputed Clebsch-Gordan
//                     terms; the term lists are built on the host from the template,
//                     once per template.
//   h_count / h_scan / h_fill  block-sparse rows of the k = 0 Hamiltonian: row block d
//                     holds the on-site block of d and, per distinct source atom s of
//                     d's incoming edges, the sum of those edges' blocks (periodic
//                     images of one pair add up), column blocks ascending.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <memory>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "so2_params.cuh"
#include "tc_ptx.cuh"

namespace {


struct LabelTables {
  int n_shells, n_orb, n_lab, lmax;
  int n_term;             // Clebsch-Gordan terms of one block (both directions have as many)
  const int* b_ptr;       // [n_orb^2 + 1] terms of each block entry ...
  const int2* b_term;     // ... (label index, coefficient as float bits)
  const int* l_ptr;       // [n_lab + 1] terms of each label ...
  const int2* l_term;     // ... (block entry index, coefficient as float bits)
};

// A template's term lists on the host: built once per template, then kept.
struct HostTables {
  std::vector<int32_t> shells;
  int n_orb = 0, n_lab = 0, lmax = 0;
  std::vector<int> bptr, lptr;       // [n_orb^2 + 1], [n_lab + 1]
  std::vector<int2> bterm, lterm;    // [n_term] each
};

// Builds the term lists of the template shell_l[0 .. n_shells).
egnn_status build_host_tables(const int32_t* shell_l, int32_t n_shells, HostTables& H) {
  int o = 0, lmax = 0, shell_off[17];
  for (int a = 0; a < n_shells; ++a) {
    const int l = shell_l[a];
    if (l < 0 || l > 3) return EGNN_ERR_UNSUPPORTED;
    if (o + 2 * l + 1 > 32) return EGNN_ERR_UNSUPPORTED;
    shell_off[a] = o;
    o += 2 * l + 1;
    lmax = 2 * l > lmax ? 2 * l : lmax;
  }
  H.shells.assign(shell_l, shell_l + n_shells);
  H.n_orb = o;
  H.lmax = lmax;
  // label order: L, then M, then k over the pairs (a, b) containing L (a outer)
  int mult[8] = {0}, lab_off[8] = {0};
  std::vector<int> kidx(n_shells * n_shells * 8, 0);
  for (int a = 0; a < n_shells; ++a)
    for (int b = 0; b < n_shells; ++b)
      for (int L = abs(shell_l[a] - shell_l[b]); L <= shell_l[a] + shell_l[b]; ++L)
        kidx[(a * n_shells + b) * 8 + L] = mult[L]++;
  int lab = 0;
  for (int L = 0; L <= lmax; ++L) {
    lab_off[L] = lab;
    lab += (2 * L + 1) * mult[L];
  }
  H.n_lab = lab;
  const int norb = o, nb = norb * norb;
  // (label, entry, coefficient) of every nonzero Clebsch-Gordan term of a block: the
  // real coupling matrices are sparse (431 of 2,025 coefficients are nonzero for the
  // {s,s,p,p,d} template), and the smallest nonzero one for l <= 3 is far above the
  // round-off left where the complex-to-real sums cancel exactly
  std::vector<int> t_lab, t_ent;
  std::vector<float> t_cg;
  for (int a = 0; a < n_shells; ++a)
    for (int b = 0; b < n_shells; ++b) {
      const int la = shell_l[a], lb = shell_l[b];
      for (int L = abs(la - lb); L <= la + lb; ++L) {
        std::vector<float> cg;
        real_cg(la, lb, L, cg);
        const int k = kidx[(a * n_shells + b) * 8 + L];
        for (int ia = 0; ia < 2 * la + 1; ++ia)
          for (int jb = 0; jb < 2 * lb + 1; ++jb)
            for (int M = 0; M < 2 * L + 1; ++M) {
              const float c = cg[(ia * (2 * lb + 1) + jb) * (2 * L + 1) + M];
              if (fabsf(c) < 1e-6f) continue;
              t_lab.push_back(lab_off[L] + M * mult[L] + k);
              t_ent.push_back((shell_off[a] + ia) * norb + shell_off[b] + jb);
              t_cg.push_back(c);
            }
      }
    }
  const int nt = (int)t_cg.size();
  // CSR by entry and by label (stable order: the sums run in a fixed order)
  std::vector<int> bptr(nb + 1, 0), lptr(lab + 1, 0);
  for (int i = 0; i < nt; ++i) {
    ++bptr[t_ent[i] + 1];
    ++lptr[t_lab[i] + 1];
  }
  for (int i = 0; i < nb; ++i) bptr[i + 1] += bptr[i];
  for (int i = 0; i < lab; ++i) lptr[i + 1] += lptr[i];
  std::vector<int2> bterm(nt), lterm(nt);
  std::vector<int> bfill(bptr.begin(), bptr.end() - 1), lfill(lptr.begin(), lptr.end() - 1);
  for (int i = 0; i < nt; ++i) {
    int2 x;
    memcpy(&x.y, &t_cg[i], 4);
    x.x = t_lab[i];
    bterm[bfill[t_ent[i]]++] = x;
    x.x = t_ent[i];
    lterm[lfill[t_lab[i]]++] = x;
  }
  H.bptr = std::move(bptr);
  H.lptr = std::move(lptr);
  H.bterm = std::move(bterm);
  H.lterm = std::move(lterm);
  return EGNN_OK;
}

// Templates whose term lists were built, most recent last (at most kTabCache).  Building
// one takes about a millisecond of host time (the Clebsch-Gordan coefficients from the
// Racah formula), longer than a conversion of a 100k-orbital structure on the GPU.
constexpr size_t kTabCache = 16;
std::mutex g_tab_mu;
std::vector<std::shared_ptr<const HostTables>> g_tab_cache;

// Copies the template's term lists into `ws` (asynchronous copies on `st` from pageable
// host memory, staged before the call returns), building them on the first call for the
// template.  An invalid template is rejected on every call and never kept.
egnn_status make_tables(const int32_t* shell_l, int32_t n_shells, LabelTables& T, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
  if (!shell_l || n_shells < 1 || n_shells > 16) return EGNN_ERR_INVALID_ARG;
  std::shared_ptr<const HostTables> H;
  {
    std::lock_guard<std::mutex> lk(g_tab_mu);
    for (const auto& c : g_tab_cache)
      if ((int)c->shells.size() == n_shells && std::equal(c->shells.begin(), c->shells.end(), shell_l)) {
        H = c;
        break;
      }
  }
  if (!H) {
    auto h = std::make_shared<HostTables>();
    const egnn_status s = build_host_tables(shell_l, n_shells, *h);
    if (s != EGNN_OK) return s;
    std::lock_guard<std::mutex> lk(g_tab_mu);
    if (g_tab_cache.size() >= kTabCache) g_tab_cache.erase(g_tab_cache.begin());
    g_tab_cache.push_back(h);
    H = h;
  }
  memset(&T, 0, sizeof(T));
  T.n_shells = n_shells;
  T.n_orb = H->n_orb;
  T.n_lab = H->n_lab;
  T.lmax = H->lmax;
  T.n_term = (int)H->bterm.size();
  const int nb = H->n_orb * H->n_orb, lab = H->n_lab, nt = T.n_term;
  const size_t o1 = ((nb + 1) * 4 + 15) & ~(size_t)15, o2 = o1 + (size_t)nt * 8;
  const size_t o3 = o2 + (((lab + 1) * 4 + 15) & ~(size_t)15), need = o3 + (size_t)nt * 8;
  if (!ws || ws_bytes < need) return EGNN_ERR_INVALID_ARG;
  char* w = (char*)ws;
  EGNN_CUDA_TRY(cudaMemcpyAsync(w, H->bptr.data(), (nb + 1) * 4, cudaMemcpyHostToDevice, st));
  EGNN_CUDA_TRY(cudaMemcpyAsync(w + o1, H->bterm.data(), (size_t)nt * 8, cudaMemcpyHostToDevice, st));
  EGNN_CUDA_TRY(cudaMemcpyAsync(w + o2, H->lptr.data(), (lab + 1) * 4, cudaMemcpyHostToDevice, st));
  EGNN_CUDA_TRY(cudaMemcpyAsync(w + o3, H->lterm.data(), (size_t)nt * 8, cudaMemcpyHostToDevice, st));
  T.b_ptr = (const int*)w;
  T.b_term = (const int2*)(w + o1);
  T.l_ptr = (const int*)(w + o2);
  T.l_term = (const int2*)(w + o3);
  return EGNN_OK;
}

// out[item][q] = sum over the terms of q of coefficient * in[item][index], for `te` items
// per group (persistent CTAs; the term list staged once per CTA when it fits).  Each
// group's inputs are contiguous in global memory and arrive by one 1-D bulk copy into
// one of two shared-memory stages, issued one group ahead; a group whose byte count is
// not a multiple of 16 (only a ragged last group can be) is loaded by all threads
// instead.  A work slot is one output q over a run of up to kRun items: q's terms are
// read once and applied to the run's items in registers; consecutive slots are
// consecutive outputs, so the stores are contiguous.  Waits are bounded (2 s); a wait
// that runs out ends every thread's loop at the same group.
// Items of a work slot.  A group of 32 items makes three runs (11, 11, 10), so the 169
// outputs of a 13-orbital template give 507 slots: two nearly full passes of 256 threads
// (runs of 16 gave 338 slots, the second pass a third full; runs of 8 cost more term
// reads per item than the fuller passes saved).
constexpr int kRun = 11;
__global__ void __launch_bounds__(256) apply_terms_kernel(const float* __restrict__ in, int nin, long long n,
                                                          const int* __restrict__ ptr, const int2* __restrict__ term,
                                                          int nout, int nterm, int staged, int te, int bulk,
                                                          float* __restrict__ out) {
  extern __shared__ __align__(16) float tsm[];
  __shared__ uint64_t full[2];
  __shared__ int abort_flag;
  const int ptr_words = staged ? ((nout + 4) & ~3) : 0;
  const int tab_words = staged ? ptr_words + 2 * ((nterm + 1) & ~1) : 0;
  int* s_ptr = reinterpret_cast<int*>(tsm);
  int2* s_term = reinterpret_cast<int2*>(s_ptr + ptr_words);
  float* stage[2] = {tsm + tab_words, tsm + tab_words + te * nin};   // [te][nin] each
  const int tid = threadIdx.x, nt = blockDim.x;
  if (tid == 0) {
    tc::mbar_init(tc::smem_u32(&full[0]), 1);
    tc::mbar_init(tc::smem_u32(&full[1]), 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (staged) {
    for (int i = tid; i <= nout; i += nt) s_ptr[i] = ptr[i];
    for (int i = tid; i < nterm; i += nt) s_term[i] = term[i];
  } else {
    s_ptr = const_cast<int*>(ptr);
    s_term = const_cast<int2*>(term);
  }
  __syncthreads();
  const long long ngroups = (n + te - 1) / te;
  // a group goes by bulk copy when its byte count is a multiple of 16
  auto by_copy = [&](long long gi) {
    return bulk && (((long long)min((long long)te, n - gi * te) * nin * 4) & 15) == 0;
  };
  auto issue = [&](long long gi, int st) {   // thread 0 only
    const uint32_t bytes = (uint32_t)(min((long long)te, n - gi * te) * nin * 4);
    const uint32_t bar = tc::smem_u32(&full[st]);
    tc::mbar_arrive_expect_tx(bar, bytes);
    tc::bulk_g2s(tc::smem_u32(stage[st]), in + gi * te * nin, bytes, bar);
  };
  uint32_t phase[2] = {0u, 0u};
  bool pend[2] = {false, false};   // thread 0: a copy into the stage is in flight
  int it = 0;
  if (tid == 0 && blockIdx.x < ngroups && by_copy(blockIdx.x)) {
    issue(blockIdx.x, 0);
    pend[0] = true;
  }
  for (long long gi = blockIdx.x; gi < ngroups; gi += gridDim.x, ++it) {
    const int st = it & 1;
    const long long g0 = gi * te;
    const int ne = (int)min((long long)te, n - g0);
    const long long gn = gi + gridDim.x;
    if (tid == 0 && gn < ngroups && by_copy(gn)) {
      issue(gn, st ^ 1);
      pend[st ^ 1] = true;
    }
    float* In = stage[st];
    if (by_copy(gi)) {
      const bool ok = tc::mbar_wait(tc::smem_u32(&full[st]), phase[st], nullptr, &abort_flag, 0);
      if (!__syncthreads_and(ok)) break;
      phase[st] ^= 1u;
      pend[st] = false;
    } else {
      for (int i = tid; i < ne * nin; i += nt) In[i] = in[g0 * nin + i];
      __syncthreads();
    }
    // work slot = (output q, run of up to kRun items): the output's terms are read once
    // and applied to the run's items held in registers; consecutive slots are
    // consecutive outputs, so each store instruction covers consecutive addresses
    const int nrun = (ne + kRun - 1) / kRun;
    float* o = out + g0 * nout;
    for (int sl = tid; sl < nout * nrun; sl += nt) {
      const int r = sl / nout, q = sl - r * nout;
      const int e0 = r * kRun, m = ne - e0 < kRun ? ne - e0 : kRun;
      float v[kRun];
#pragma unroll
      for (int i = 0; i < kRun; ++i) v[i] = 0.f;
      const int t1 = s_ptr[q + 1];
      for (int t = s_ptr[q]; t < t1; ++t) {
        const int2 tm = s_term[t];
        const float cf = __int_as_float(tm.y);
        const float* x = In + e0 * nin + tm.x;
#pragma unroll
        for (int i = 0; i < kRun; ++i)
          if (i < m) v[i] = fmaf(cf, x[i * nin], v[i]);
      }
#pragma unroll
      for (int i = 0; i < kRun; ++i)
        if (i < m) o[(size_t)(e0 + i) * nout + q] = v[i];
    }
    __syncthreads();   // stage st is free for the copy issued in the next iteration
  }
  // a copy still in flight (only after a wait ran out) must land before the CTA exits
  if (tid == 0) {
    for (int st = 0; st < 2; ++st) {
      if (!pend[st]) continue;
      const uint64_t t0 = tc::globaltimer();
      while (!tc::mbar_try_wait(tc::smem_u32(&full[st]), phase[st]) && tc::globaltimer() - t0 < 2000000000ull) {
      }
    }
  }
}

cudaError_t launch_terms(const float* in, int nin, long long n, const int* ptr, const int2* term, int nout,
                         int nterm, float* out, cudaStream_t st) {
  const size_t tab_full = 4 * (size_t)((nout + 4) & ~3) + 8 * (size_t)((nterm + 1) & ~1);
  const int staged = tab_full <= 32 * 1024 ? 1 : 0;
  const size_t tab = staged ? tab_full : 0;
  // items per group: two stages, four CTAs per SM within ~55 KB of shared memory each,
  // else two within ~110 KB
  auto bytes = [&](int te) { return tab + 2 * (size_t)te * nin * 4; };
  int te = 32;
  while (te > 4 && bytes(te) > 55 * 1024) te >>= 1;
  while (te > 1 && bytes(te) > 110 * 1024) te >>= 1;
  const int bulk = (((uintptr_t)in & 15) == 0 && te % 4 == 0) ? 1 : 0;
  const size_t sm = bytes(te);
  cudaError_t err = cudaFuncSetAttribute(apply_terms_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (err != cudaSuccess) return err;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const long long groups = (n + te - 1) / te;
  const int grid = (int)(groups < 4LL * nsm ? groups : 4LL * nsm);
  apply_terms_kernel<<<grid, 256, sm, st>>>(in, nin, n, ptr, term, nout, nterm, staged, te, bulk, out);
  return cudaGetLastError();
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
  // run k of block j (-1: on-site only) and its column
  auto block_of = [&](int j, int& k, int& col) {
    if (j < n_lo) {
      k = j;
      col = run_s[k];
    } else if (j == n_lo) {
      k = self_run;
      col = d;
    } else {
      k = j - 1 + (self_run >= 0 ? 1 : 0);
      col = run_s[k];
    }
  };
  for (int j = tid; j < nblk; j += blockDim.x) {
    int k, col;
    block_of(j, k, col);
    bsr_col[row0 + j] = col;
  }
  // all nblk * nb output elements of the row block (contiguous in bsr_val), kU per
  // thread per pass: the on-site term and the first edge of all kU elements are loaded
  // before any is summed, so kU loads per thread are in flight (a run is mostly one
  // edge).  Each element sums on-site, then its run's edges in edge order.
  constexpr int kU = 4;
  const int tot = nblk * nb;
  float* out = bsr_val + (size_t)row0 * nb;
  for (int i0 = tid; i0 < tot; i0 += kU * blockDim.x) {
    float a[kU], v[kU];
    int kk[kU], qq[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * (int)blockDim.x;
      a[u] = 0.f;
      v[u] = 0.f;
      kk[u] = -1;
      qq[u] = 0;
      if (i < tot) {
        const int j = i / nb, q = i - j * nb;
        int k, col;
        block_of(j, k, col);
        kk[u] = k;
        qq[u] = q;
        if (col == d) a[u] = onsite[(size_t)d * nb + q];
        if (k >= 0) v[u] = edge_blocks[(size_t)run_b[k] * nb + q];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * (int)blockDim.x;
      if (i >= tot) continue;
      const int k = kk[u];
      float x = a[u];
      if (k >= 0) {
        x += v[u];
        for (int e = run_b[k] + 1; e < run_b[k + 1]; ++e) x += edge_blocks[(size_t)e * nb + qq[u]];
      }
      out[i] = x;
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
  EGNN_CUDA_TRY(launch_terms(labels, T.n_lab, n, T.b_ptr, T.b_term, T.n_orb * T.n_orb, T.n_term, blocks, st));
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
  EGNN_CUDA_TRY(launch_terms(blocks, T.n_orb * T.n_orb, n, T.l_ptr, T.l_term, T.n_lab, T.n_term, labels, st));
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
