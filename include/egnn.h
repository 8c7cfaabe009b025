/*
 * egnn.h -- C ABI of libegnn.so: the data-parallel hot path of an SO(2)-equivariant
 * (eSCN) message-passing layer for electronic-structure prediction, on one
 * NVIDIA B200 (sm_100a).
 *
 * Sources (page title, section):
 *   [MALOQ]  "MALOQ: Massively Accelerated Learning of Operators for Quantum
 *            Transport" (arXiv 2606.28911).
 *   [DEGNN]  review page of "Distributed Equivariant Graph Neural Networks for
 *            Large-Scale Electronic Structure Prediction" (arXiv 2507.03840).
 *
 * Conventions shared by every call
 *   - Every pointer named "device" is CUDA device memory owned by the caller.
 *     The library allocates nothing (no cudaMalloc, no library allocator): all
 *     scratch comes from the caller's `workspace`, sized by egnn_workspace_bytes,
 *     except in egnn_build_graph_noalloc (a fixed array in the library's module).
 *   - Work is launched on `cuda_stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Calls are asynchronous unless stated otherwise.
 *   - Host-checkable errors (null pointers, unsupported sizes, workspace too
 *     small) are returned before anything is launched.
 *   - Device-side checks (an index out of range, a bounded wait that ran out)
 *     never trap: the kernel writes a non-zero code into the graph's `status`
 *     word and skips the access; egnn_read_status reports it.
 *   - Real spherical-harmonic basis, orthonormal, no Condon-Shortley phase,
 *     coefficient index l*l + l + m (m = -l..l); Y_1 is proportional to (y,z,x).
 *   - Embedding layout [n_atoms][(lmax+1)^2][C], C contiguous.
 */
#ifndef EGNN_H
#define EGNN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  EGNN_OK = 0,
  EGNN_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad box/rcut       */
  EGNN_ERR_CAPACITY = 2,      /* graph arrays too small: n_edges holds the need   */
  EGNN_ERR_UNSUPPORTED = 3,   /* lmax/mmax/C/heads/dtype/template outside limits  */
  EGNN_ERR_CUDA = 4,          /* a CUDA runtime call failed                        */
  EGNN_ERR_DEVICE_CHECK = 5   /* a kernel set the status word (see egnn_read_status) */
} egnn_status;

/* Values of the device status word (egnn_graph::status; first writer wins). */
enum {
  EGNN_DEV_BAD_POSITION = 1,      /* a coordinate outside [0, box) or not finite        */
  EGNN_DEV_SEGMENT_TOO_LARGE = 2, /* an atom with more than 4096 incoming edges         */
  EGNN_DEV_INDEX_RANGE = 3,       /* a source index outside [0, n_atoms)                */
  EGNN_DEV_COUNT_MISMATCH = 4,    /* neighbour count and fill passes disagreed           */
  EGNN_DEV_EDGE_OVERFLOW = 5,     /* more than 2^31 - 1 edges                            */
  EGNN_DEV_WAIT_TIMEOUT = 6,      /* a bounded wait of a pipelined kernel ran out        */
  EGNN_DEV_BAD_GRAPH = 7          /* row_ptr not monotone or out of range                */
};

typedef enum { EGNN_FP32 = 0, EGNN_BF16 = 1 } egnn_dtype;

/* Layer hyper-parameters.  Limits: 0 <= mmax <= min(lmax, 2), lmax <= 6,
 * channels in {16, 32, 64, 128} (multiple of heads), 1 <= heads <= 16,
 * 2 <= n_rbf <= 64, rcut > 0.  dtype EGNN_FP32: fp32 embeddings, weights and
 * arithmetic (no TF32).  EGNN_BF16: bf16 embeddings and weights, fp32
 * accumulation, bf16 output. */
typedef struct {
  int32_t lmax, mmax, channels, heads, n_rbf;
  float rcut;
  int32_t dtype;
} egnn_layer_desc;

/* Destination-sorted ("incoming edge") graph, [DEGNN] "What carries the
 * argument": atom d owns every edge s -> d.  All arrays are device memory
 * owned by the caller.  Wigner layout per edge e: for l = 0..lmax, the rows
 * m = -min(l,mmax)..min(l,mmax) of D^l(R_e), each row m' = -l..l, row-major,
 * l-blocks concatenated: egnn_wigner_floats(lmax, mmax) floats per edge.
 * R_e is the rotation taking r_e = x_s + shift*box - x_d onto +z
 * ([MALOQ] Section III-C1 and Fig. 3 rotate every edge to one common axis). */
typedef struct {
  int32_t n_atoms;
  int32_t lmax, mmax;       /* set by egnn_build_graph: Wigner rows stored      */
  int64_t capacity;         /* edges the per-edge arrays can hold               */
  int64_t n_edges;          /* written by egnn_build_graph                       */
  int32_t* row_ptr;         /* [n_atoms + 1]                                      */
  int32_t* src;             /* [capacity]  source atom of each edge              */
  int8_t* shift;            /* [capacity][3] periodic image of the source        */
  float* dist;              /* [capacity]  |r_e|                                  */
  float* wigner;            /* [capacity][egnn_wigner_floats(lmax, mmax)]       */
  int32_t* status;          /* [1] device status word, 0 = ok; cleared by build  */
} egnn_graph;

/* Floats of Wigner data stored per edge: sum_l (2 min(l,mmax) + 1)(2l + 1). */
int32_t egnn_wigner_floats(int32_t lmax, int32_t mmax);

/* Which call a workspace is for. */
enum {
  EGNN_WS_BUILD_GRAPH = 0,
  EGNN_WS_LAYER = 1,
  EGNN_WS_HAMILTONIAN = 2,
  EGNN_WS_LABELS = 3,       /* egnn_labels_to_blocks / egnn_blocks_to_labels (1 MB)   */
  EGNN_WS_ASSEMBLY = 4      /* egnn_assemble_hamiltonian (4 bytes per atom)          */
};

/* Bytes of device workspace `which` needs (0 allowed).  For EGNN_WS_BUILD_GRAPH
 * only n_atoms matters and desc may be NULL.  Tensor-core calls (bf16, C = 128), with
 * L = lmax + 1:
 *   layer: no per-edge message is stored.  The size grows with n_edges only by two
 *     partial-softmax records per tile of 128 edges and a 4-byte destination index
 *     per edge, 2 * 4 (L^2 C + 32) / 128 + 4 bytes per edge (206 at lmax 4), and
 *     with n_atoms by an fp32 accumulator of L^2 C values per atom;
 *   head: grows with n_edges by the per-edge record of the SO(2) outputs
 *     (4 L C + 4 C sum_{b=1..mmax} (L - b) bytes, 6 KB at lmax 4, mmax 2);
 * the gate and A-operand buffers of both are sized for one range of at most 4096
 * edge tiles and stop growing beyond it. */
size_t egnn_workspace_bytes(int32_t which, const egnn_layer_desc* desc, int32_t n_atoms,
                            int64_t n_edges);

/*
 * egnn_build_graph -- periodic radius graph (cell list) -> destination CSR,
 * then per-edge distance and Wigner-D rows.
 *   [MALOQ] Section I and Table II (atoms within a cutoff, degrees of hundreds),
 *   Section III ("Compute Wigners", once per structure), Section III-C1.
 * pos      device fp64 [n_atoms][3], every coordinate in [0, box_k).
 * species  device int32 [n_atoms] (validated >= 0; the layer does not use it).
 * box      host fp64 [3], orthorhombic periodic cell lengths.
 * rcut     cutoff in the units of pos; an edge s -> d (s may equal d for a
 *          non-zero shift) exists iff, in fp64 with separately rounded
 *          operations, r = (x_s + shift*box) - x_d and
 *          ((r.x*r.x + r.y*r.y) + r.z*r.z) < rcut*rcut.
 * Segments are sorted by (s, shift.x, shift.y, shift.z) ascending, so the list
 * is unique.  lmax/mmax select the Wigner rows to store (limits as for layers).
 * Synchronises `cuda_stream` once to read the edge count.  If g->capacity is
 * smaller than the count, returns EGNN_ERR_CAPACITY with g->n_edges set and
 * row_ptr filled; the caller grows the arrays and calls again.
 * Limits: n_atoms >= 1; at most 4096 incoming edges per atom.
 */
egnn_status egnn_build_graph(const double* pos, const int32_t* species, int32_t n_atoms,
                             const double box[3], double rcut, int32_t lmax, int32_t mmax,
                             egnn_graph* g, void* workspace, size_t ws_bytes, void* cuda_stream);

/*
 * egnn_edge_geometry -- recompute every edge's distance and Wigner-D rows of an
 * existing graph for new positions, keeping its neighbour list (row_ptr, src, shift),
 * e.g. when atoms moved less than a skin distance since the list was built.
 *   [MALOQ] Section III-C1 and Fig. 3 (the per-edge rotation to a common axis).
 * pos  device fp64 [g->n_atoms][3], wrapped into the box as for egnn_build_graph;
 * box  host fp64 [3].  Degrees stored as g->lmax / g->mmax.  Asynchronous; does not
 * clear the status word.  A source index outside [0, n_atoms) sets it to
 * EGNN_DEV_INDEX_RANGE (that edge's rows are left unwritten).
 */
egnn_status egnn_edge_geometry(const double* pos, const double box[3], egnn_graph* g, void* cuda_stream);

/*
 * egnn_build_graph_noalloc -- egnn_build_graph without a caller-supplied workspace.
 * The pages have no counterpart to this call; it exists for callers that cannot
 * obtain device memory for a workspace, for example a component that only
 * receives device pointers from its host application and may not call
 * cudaMalloc itself, or a loop that forbids allocation after start-up.  It makes
 * no allocation of any kind: its scratch is a fixed array of about 4.7 MB in the
 * library's device memory, one copy on every GPU that loads the library, held
 * until the process exits.
 * Arguments, outputs and errors are those of egnn_build_graph, plus:
 *   n_atoms above 131072 returns EGNN_ERR_UNSUPPORTED before any work;
 *   the first call on a device looks up the array's device address (once per
 *   device, with that device current) and keeps it for the life of the process;
 *   make that first call before any stream capture.  The kept address belongs to
 *   the device's context at that time: after cudaDeviceReset (or any teardown of
 *   the primary context) do not call this entry point again in the same process.
 * All calls share the one array (whatever stream they use) and the kernels clear
 * what must start at zero, so calls that overlap on the GPU race: order them, for
 * example on one stream.
 */
egnn_status egnn_build_graph_noalloc(const double* pos, const int32_t* species, int32_t n_atoms,
                                     const double box[3], double rcut, int32_t lmax, int32_t mmax,
                                     egnn_graph* g, void* cuda_stream);

/*
 * egnn_layer_forward -- one eSCN message-passing layer in the incoming-edge layout.
 *   [MALOQ] Sections II-B1 and III (rotate each edge to a common axis, SO(2)
 *   constrained linear layers, aggregate onto the target node), III-D and
 *   Fig. 4(b) (message from the concatenated pair); [DEGNN] "What carries the
 *   argument" (attention and aggregation local to the owner of the edges).
 * For every atom d and incoming edge e = (s -> d):
 *   z = [n_s || n_d] (2C channels); x[l,m,:] = g_e[l,:] * (D^l(R_e) z^l)[m,:]
 *   for |m| <= mmax, with g_e = W2 SiLU(W1 rho(|r_e|) + b1) + b2 and
 *   rho_k(r) = exp(-(r - k rcut/(K-1))^2 / (2 (rcut/(K-1))^2));
 *   y0 = W0 x0;  y+m = Wm1 x+m - Wm2 x-m,  y-m = Wm2 x+m + Wm1 x-m  (x+-m stacked
 *   over l = m..lmax);  a_{e,h} = A[h,:] . SiLU(y0) + bA[h];
 *   msg_e^l = (kept rows of D^l(R_e))^T y^l;
 *   out_d = n_d + sum_e softmax_e(a_{e,h(c)}) msg_e, head h(c) = c / (C/heads).
 * weights  device, packed row-major ([out][in]) in this order, dtype per desc:
 *   W1[C][K] b1[C] W2[(lmax+1)2C][C] b2[(lmax+1)2C] W0[(lmax+1)C][(lmax+1)2C]
 *   then for m = 1..mmax: Wm1[n_m C][n_m 2C] Wm2[n_m C][n_m 2C] (n_m = lmax+1-m)
 *   then A[heads][(lmax+1)C] bA[heads].
 *   Input index of x0 is l*2C + c2, of x+-m is (l-m)*2C + c2; output index of y0
 *   is l*C + c, of y+-m is (l-m)*C + c; gate index l*2C + c2.
 * node_in / node_out  device [n_atoms][(lmax+1)^2][C], fp32 or bf16 per dtype;
 *   their byte ranges must be disjoint (any overlap, partial included, returns
 *   EGNN_ERR_INVALID_ARG).  An atom without incoming edges gets out = in.
 *   weights, node_in and node_out must be 16-byte aligned (EGNN_ERR_INVALID_ARG).
 * g must come from egnn_build_graph with the same lmax/mmax and rcut.
 */
egnn_status egnn_layer_forward(const egnn_graph* g, const egnn_layer_desc* desc,
                               const void* weights, const void* node_in, void* node_out,
                               void* workspace, size_t ws_bytes, void* cuda_stream);

/*
 * egnn_hamiltonian_blocks -- off-diagonal Hamiltonian block of every directed edge.
 *   [MALOQ] Section III-B1 and Eq. (1) (block H^{ab} = CG image of labels |L,M>,
 *   L = |l_a - l_b|..l_a + l_b), Section III-B2 (orbital template, one block per
 *   edge), Section III (edge blocks use the messages directly).
 * Per edge: t = the gated SO(2) message above computed with the head's own
 * weights (no attention, no aggregation); labels h[L,M,k] = sum_c U^L[k][c] t[L,M,c]
 * with one k per shell pair (a, b) containing L (pairs lexicographic, a outer);
 * block[(a,i),(b,j)] = sum_{L,M} C^L_{(l_a i)(l_b j),M} h[L,M,k(a,b,L)], where C^L
 * is the real Clebsch-Gordan matrix of the basis above (orthonormal columns,
 * first non-zero entry of column M=-L positive).  The tensor-core path applies U^L
 * in the edge frame (U^L folded into the SO(2) weights, then the labels rotated
 * back), which equals the order above up to rounding because U^L mixes channels
 * only and the rotation mixes m only.
 * head_weights device, packed like a layer's W1..Wm2 (no A, bA), then U^L[mult_L][C]
 *   for L = 0..lmax (absent when mult_L = 0).
 * shell_l   host int32 [n_shells]: orbital template shared by all species,
 *   e.g. {0,0,1,1,2}; every l_a + l_b <= lmax, every l_a <= 3, n_orb <= 32.
 * node_emb  device [n_atoms][(lmax+1)^2][C] (dtype per desc).
 * blocks    device fp32 [n_edges][n_orb][n_orb]; rows are the destination atom's
 *   orbitals, columns the source atom's.
 */
egnn_status egnn_hamiltonian_blocks(const egnn_graph* g, const egnn_layer_desc* desc,
                                    const void* head_weights, const int32_t* shell_l,
                                    int32_t n_shells, const void* node_emb, float* blocks,
                                    void* workspace, size_t ws_bytes, void* cuda_stream);

/* egnn_check_bounded_wait -- diagnostic of the failure path (the pages have no
 * counterpart).  Every pipelined kernel waits on mbarriers with a time limit and, when
 * the limit runs out, records EGNN_DEV_WAIT_TIMEOUT in the status word and returns
 * instead of hanging.  This call runs that same wait routine in a one-thread kernel on
 * an mbarrier that nothing arrives on, with a limit of `limit_us` microseconds
 * (1 .. 2,000,000), so the status word of `g` reads EGNN_DEV_WAIT_TIMEOUT afterwards.
 * Asynchronous on `cuda_stream`; the context stays usable. */
egnn_status egnn_check_bounded_wait(egnn_graph* g, uint32_t limit_us, void* cuda_stream);

/*
 * Label <-> block conversion ([MALOQ] Section III-B1, Eq. (1); Section III-B2 and
 * Fig. 2(b-d): Matrix -> Label for training targets, Label -> Matrix for the
 * prediction, on the GPU, driven by the orbital template).
 * Orbital template: shell_l host int32 [n_shells] (1..16 shells, each l <= 3, at most
 * 32 orbitals), shared by both atoms of a block.  Labels per block: for L = 0 .. 2 max l,
 * M = -L..L, then k over the shell pairs (a, b) with |l_a - l_b| <= L <= l_a + l_b
 * (lexicographic, a outer): the layout egnn_hamiltonian_blocks uses.  Label
 * h[L, M, k] = sum_{i, j} C^L_{(l_a i)(l_b j), M} H[(a, i), (b, j)] with the real
 * Clebsch-Gordan matrices of egnn_hamiltonian_blocks; since each C^L has orthonormal
 * columns and together they are square per pair, the two calls are inverse.
 * blocks device fp32 [n][n_orb][n_orb]; labels device fp32 [n][egnn_label_count(...)].
 * workspace: egnn_workspace_bytes(EGNN_WS_LABELS, ...) bytes of device memory (tables).
 * Asynchronous on `cuda_stream`.  Errors: bad template EGNN_ERR_UNSUPPORTED, null
 * pointers or small workspace EGNN_ERR_INVALID_ARG.
 */
int32_t egnn_label_count(const int32_t* shell_l, int32_t n_shells);
egnn_status egnn_blocks_to_labels(const float* blocks, int64_t n, const int32_t* shell_l, int32_t n_shells,
                                  float* labels, void* workspace, size_t ws_bytes, void* cuda_stream);
egnn_status egnn_labels_to_blocks(const float* labels, int64_t n, const int32_t* shell_l, int32_t n_shells,
                                  float* blocks, void* workspace, size_t ws_bytes, void* cuda_stream);

/*
 * egnn_assemble_hamiltonian -- the k = 0 Hamiltonian of the structure as block-sparse
 * rows (BSR) from on-site and per-edge orbital blocks ([MALOQ] Section III-B2, the
 * Label -> Matrix reconstruction of the whole matrix; [DEGNN] one matrix of 104,833
 * orbitals for the 8,064-atom cell).
 * Row block d (orbitals of atom d) holds the on-site block onsite[d] at column d and,
 * for every distinct source atom s of d's incoming edges, the sum of those edges'
 * blocks at column s (periodic images of one pair add up; images of d itself add to
 * the on-site block).  Column blocks ascend within a row; sums run in edge order, so
 * the result is deterministic.
 * onsite device fp32 [n_atoms][n_orb][n_orb]; edge_blocks device fp32
 * [n_edges][n_orb][n_orb] in the graph's edge order (e.g. from egnn_hamiltonian_blocks).
 * bsr_row_ptr device int32 [n_atoms + 1]; bsr_col device int32 [capacity]; bsr_val device
 * fp32 [capacity][n_orb][n_orb].  capacity >= n_atoms + n_edges is required (else
 * EGNN_ERR_CAPACITY) and always suffices; the block count is bsr_row_ptr[n_atoms].
 * workspace: egnn_workspace_bytes(EGNN_WS_ASSEMBLY, NULL, n_atoms, 0) bytes.  Asynchronous.
 */
egnn_status egnn_assemble_hamiltonian(const egnn_graph* g, const float* onsite, const float* edge_blocks,
                                      int32_t n_orb, int32_t* bsr_row_ptr, int32_t* bsr_col, float* bsr_val,
                                      int64_t capacity, void* workspace, size_t ws_bytes, void* cuda_stream);

/* Synchronises `cuda_stream`, returns EGNN_ERR_DEVICE_CHECK if the graph's status
 * word is non-zero (its value goes to *code when code != NULL), else EGNN_OK. */
egnn_status egnn_read_status(const egnn_graph* g, int32_t* code, void* cuda_stream);

/* Short text for a status value (static storage). */
const char* egnn_status_string(egnn_status s);

/*
 * egnn_profile / egnn_profile_read -- opt-in timing of the main kernel of tensor-core
 * egnn_layer_forward calls, the fused SO(2) layer kernel (one launch per range of at
 * most 4096 edge tiles); a diagnostic, the pages have no counterpart.
 * egnn_profile(1) clears the record and starts recording; egnn_profile(0) stops.
 * While recording, every such launch of a layer call is bracketed by two CUDA
 * events recorded on that call's stream (at most 4096 launches per record; later
 * ones are not recorded).  The events are created on first use, on the device
 * current at the time, and kept until the process exits: use one device per
 * process.  Not thread-safe.  Head calls and the SIMT path are not recorded.
 * egnn_profile_read waits for the recorded events and returns the summed launch
 * time in milliseconds, the number of launches and the number of edges they
 * processed; null outputs return EGNN_ERR_INVALID_ARG, a CUDA error EGNN_ERR_CUDA.
 */
egnn_status egnn_profile(int32_t enable);
egnn_status egnn_profile_read(double* gemm_ms, int64_t* launches, int64_t* edges);

#ifdef __cplusplus
}
#endif
#endif /* EGNN_H */
