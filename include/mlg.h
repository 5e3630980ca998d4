/*
 * mlg.h -- C ABI of the B200 neighbour-graph library (libmlg.so).
 *
 * Two stages of machine-learned interatomic potential inference, entirely on
 * one GPU:
 *
 *   1. mlg_build_csr: an O(N) cell-list search for every periodic neighbour
 *      image within rcut, emitted as a destination-sorted CSR edge list
 *      (row_ptr, source index, integer image shift, edge vector, distance,
 *      smooth switch s(r)).  It replaces the host-side edge construction and
 *      the host-to-device copies that the deepmd-kit issue "DPA4 .pt2 LAMMPS
 *      (C++ AOTI) inference 3-6x slower than Python (ASE) due to CPU-side
 *      edge construction and data marshalling" measures as the bottleneck
 *      (Root cause analysis, bottlenecks 1 and 2: createEdgeTensors() and the
 *      synchronising copies), and it produces the destination CSR
 *      (destination_order / destination_row_ptr) that the deepmd-kit issue
 *      "NeighborGraph attention is 4-9x slower than dense and OOM-prone --
 *      move to block-dense attention via the destination CSR" builds on
 *      (Proposed fix).
 *
 *   2. mlg_block_attention: block-dense multi-head attention of every centre
 *      over its own edges (NeighborGraph issue, Proposed fix: each centre's
 *      edges form one small dense block, found by destination_row_ptr; the
 *      block is attended to with dense products, unequal row lengths masked
 *      per row, and the outputs go back to their edges; no (sum nnei^2, c)
 *      pair-axis tensor ever exists).
 *
 *   mlg_forward runs stage 1 and then n_layers of stage 2.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named "device" are CUDA device pointers (e.g. the data_ptr()
 *    of a torch CUDA tensor); they are owned by the caller, never freed or
 *    retained by the library.  Structs passed by pointer are read during the
 *    call only (host memory).
 *  - Every call is asynchronous and stream-ordered on `stream` (a
 *    cudaStream_t; NULL = the legacy default stream).  The library never
 *    synchronises, never allocates device or pinned memory, keeps no state
 *    between calls and may be called from several host threads on different
 *    streams with different workspaces.
 *  - The return value is the host-side status (mlg_status): argument and
 *    workspace checks, and the launch result (cudaGetLastError).  Errors that
 *    depend on device data are OR-ed into the device word csr->status
 *    (mlg_status_bits); read it after synchronising the stream.
 *  - Coordinates and geometry are fp64 always.  Attention features and
 *    weights are fp32 (MLG_F32) or fp64 (MLG_F64).
 */
#ifndef MLG_H
#define MLG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the runtime's opaque stream handle). */
typedef struct CUstream_st* mlg_stream_t;

/* Host-side return codes. */
typedef enum {
    MLG_OK = 0,
    MLG_ERR_INVALID_ARG = 1,  /* a NULL pointer, a non-positive size, rcut <= r_on, a non-finite box */
    MLG_ERR_WORKSPACE = 2,    /* ws_bytes smaller than the matching *_workspace_bytes() */
    MLG_ERR_CAPACITY = 3,     /* capacity < 0 */
    MLG_ERR_INPUT_DATA = 4,   /* reserved for host-visible data errors */
    MLG_ERR_UNSUPPORTED = 5,  /* a shape the library does not handle (see each call) */
    MLG_ERR_CUDA = 6          /* a CUDA launch error (cudaGetLastError) */
} mlg_status;

/* Bits OR-ed into the device word csr->status. */
typedef enum {
    MLG_STATUS_NONFINITE_COORD = 1u, /* an atom had a NaN/Inf coordinate; it has no edges */
    MLG_STATUS_TYPE_RANGE = 2u,      /* a type outside [0, n_types) */
    MLG_STATUS_CAPACITY = 4u,        /* E > capacity: row_ptr and n_edges are complete,
                                        edges at index >= capacity were not written,
                                        attention skipped */
    MLG_STATUS_IMAGE_RANGE = 8u,     /* an atom lies more than 511 box lengths outside the
                                        box along a periodic axis; it was left out */
    MLG_STATUS_TIES = 16u,           /* reserved (no longer raised: ties at the cap are
                                        broken exactly by (source, shift)) */
    MLG_STATUS_INTERNAL = 32u,       /* the count and fill passes disagreed on a row (never
                                        expected); that row is incomplete */
    MLG_STATUS_TIMEOUT = 64u,        /* a bounded wait ran out (never expected in normal
                                        use); the output of that call is incomplete */
    MLG_STATUS_ROW_TOO_LONG = 128u,  /* an attention call met a destination with more edges
                                        than the nnei_max it was given; that destination's
                                        output rows were not written */
    MLG_STATUS_LIST_INCOMPLETE = 256u /* mlg_verlet_step: the candidate list misses pairs
                                        (a destination had more than 256 candidates within
                                        rcut + skin, or the list's capacity was too small);
                                        the refined CSR may miss edges */
} mlg_status_bits;

/* Arithmetic type of attention features and weights. */
typedef enum { MLG_F32 = 0, MLG_F64 = 1 } mlg_dtype;

/* The atomic system (DPA4 LAMMPS issue, Reproduction: coordinates as double,
 * atom types; the box and periodicity of the simulation cell). */
typedef struct {
    int64_t n_atoms;        /* N >= 1 */
    const double* coords;   /* device [N][3], Angstrom; any values (need not be wrapped) */
    const int32_t* types;   /* device [N] or NULL; validated into MLG_STATUS_TYPE_RANGE,
                               not used by the attention */
    int32_t n_types;        /* >= 1 when types != NULL */
    double box[9];          /* HOST, row-major rows a1, a2, a3 (Angstrom).  Every entry must be
                               finite.  Along a periodic axis k the row a_k must be (0..L_k..0)
                               with L_k > 0 (orthorhombic cells; a sheared cell returns
                               MLG_ERR_UNSUPPORTED).  Rows of open axes are not used for
                               images (the shift is 0 there). */
    uint8_t pbc[3];         /* HOST, 1 = periodic along axis k, 0 = open */
} mlg_system;

/* The destination CSR (NeighborGraph issue, Proposed fix: destination_order /
 * destination_row_ptr).  All arrays are caller-owned DEVICE memory.
 *
 * Edges of destination i are rows [row_ptr[i], row_ptr[i+1]).  Inside a
 * destination they are in canonical order of (source, shift x, shift y,
 * shift z), ascending.  A destination with more than nnei_max in-cutoff
 * neighbours keeps the nnei_max nearest, ties broken by (source, shift).
 * For edge e of destination i with source j and shift S:
 *   vec[e]  = (x_j + S_0 a1 + S_1 a2 + S_2 a3) - x_i,   fp64, rounded per op
 *   dist[e] = |vec[e]| < rcut,                          fp64, IEEE sqrt
 *   sw[e]   = s(dist): 1 below r_on, 0.5 (1 + cos(pi u)) with
 *             u = (dist - r_on) / (rcut - r_on) up to rcut.
 * N * nnei_max rows always suffice for `capacity`. */
typedef struct {
    int64_t capacity;       /* rows available in src/shift/vec/dist/sw (and in attention G) */
    int64_t* row_ptr;       /* [N + 1] */
    int32_t* src;           /* [capacity] */
    int32_t* shift;         /* [capacity][3] */
    double* vec;            /* [capacity][3] */
    double* dist;           /* [capacity] */
    double* sw;             /* [capacity] */
    int64_t* n_edges;       /* device scalar: E = row_ptr[N] */
    int64_t* n_truncated;   /* device scalar: destinations with more than nnei_max neighbours */
    uint32_t* status;       /* device scalar: mlg_status_bits */
} mlg_csr;

/* Bytes of device workspace that mlg_build_csr needs for this system.  The
 * cell grid depends on N, rcut, the box and pbc (not on the coordinates).
 * For systems built by the kernel chain (more than 4,096 atoms, or narrow
 * boxes aside) the size includes 516 bytes per atom in which the count pass
 * keeps the accepted keys of every row of at most 64 of them, so that the
 * fill pass does not search the stencil again.  Returns 0 for invalid
 * arguments. */
size_t mlg_build_csr_workspace_bytes(int64_t n_atoms, double rcut, const double box[9],
                                     const uint8_t pbc[3]);

/* Build the destination CSR of `sys` (see mlg_csr).  Resets *csr->status,
 * *csr->n_truncated; writes row_ptr, n_edges and min(E, capacity) edges.
 *   rcut      cutoff radius (> r_on > 0); strict r < rcut
 *   r_on      onset of the cosine switch
 *   nnei_max  per-destination cap (sel), 1..256, else MLG_ERR_UNSUPPORTED
 *   ws        device workspace of ws_bytes >= mlg_build_csr_workspace_bytes(), 256-byte aligned
 * The result is deterministic: bitwise identical across calls, streams and GPUs. */
int mlg_build_csr(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                  const mlg_csr* csr, void* ws, size_t ws_bytes, mlg_stream_t stream);

/* Several independent systems in one CSR (batched inference of many
 * structures, as the NValchemi batching on the source pages does; there is
 * no neighbour cache, so a refill of the same size, a cell change or a new
 * partition always gives the fresh graph).  Atom a of system k is centre and
 * source number off_k + a, off_k = the atoms of systems 0..k-1; rows of
 * system k are its mlg_build_csr rows with sources offset by off_k, in that
 * order, so row_ptr has sum(N_k) + 1 entries.  Systems never pair with each
 * other; each has its own box, pbc and types.  A system with 0 atoms adds no
 * rows.  Same outputs, status bits and capacity behaviour as mlg_build_csr;
 * arguments as there, plus:
 *   systems    host array of n_systems descriptors (device coordinates)
 *   ws         >= mlg_build_csr_batch_workspace_bytes(), 256-byte aligned
 * The systems run one after another on `stream` (a launch chain per system,
 * with one scan of all kept counts between the count and fill passes). */
size_t mlg_build_csr_batch_workspace_bytes(const mlg_system* systems, int32_t n_systems,
                                           double rcut);
int mlg_build_csr_batch(const mlg_system* systems, int32_t n_systems, double rcut, double r_on,
                        int32_t nnei_max, const mlg_csr* csr, void* ws, size_t ws_bytes,
                        mlg_stream_t stream);

/* Bytes of device workspace that mlg_block_attention needs (0: it needs none). */
size_t mlg_attention_workspace_bytes(int64_t n_centres, int32_t nnei_max, int32_t channels,
                                     int32_t heads, mlg_dtype dtype);

/* One block-dense attention layer over every destination of `csr`.
 *   G_in, G_out  device [capacity][channels] in CSR edge order, dtype; rows >= E are not
 *                touched.  G_out must not alias G_in.
 *   Wq, Wk, Wv   device [channels][channels] row-major, y = x W (q = g Wq)
 *   channels % heads == 0; head size d = channels / heads <= 64; channels <= 256
 * Per destination i with n edges (rows a, b < n), per head h (columns h d .. h d + d):
 *   l_ab = s_a s_b (q_a . k_b) / sqrt(d);  P_ab = exp(l_ab - max_b l) / sum_b exp(...);
 *   G_out[a, h d + t] = sum_b P_ab v_b[t].
 * Slots beyond a destination's n edges do not exist (masked).  Reads E from csr->row_ptr
 * on the device; if *csr->status has MLG_STATUS_CAPACITY set, nothing is written.
 * nnei_max is normally the cap the CSR was built with.  A destination with more than
 * nnei_max edges is skipped on every kernel path: its output rows are left as they were
 * and MLG_STATUS_ROW_TOO_LONG is OR-ed into *csr->status. */
int mlg_block_attention(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                        int32_t channels, int32_t heads, mlg_dtype dtype, const void* G_in,
                        void* G_out, const void* Wq, const void* Wk, const void* Wv, void* ws,
                        size_t ws_bytes, mlg_stream_t stream);

/* One attention layer with the slot-occupancy ("smooth") softmax (NeighborGraph
 * issue, Numerics note: empty slots counted as phantoms in the denominator; the
 * weights factor as w_b = softmax_b * sum_b e_b / D~).  As mlg_block_attention,
 * plus phi = nnei_max - n phantom slots per destination: the zero-padded
 * slots of the dense (nloc, nnei_max, c) route, left unmasked, whose logit is
 * exactly 0 and whose value is 0:
 *   m_a = max(max_b l_ab, 0 if phi > 0),  D~ = sum_b exp(l_ab - m_a) + phi exp(-m_a),
 *   G_out[a, h d + t] = sum_b exp(l_ab - m_a) v_b[t] / D~.
 * Destinations with more than nnei_max edges are left untouched and flagged with
 * MLG_STATUS_ROW_TOO_LONG.  Runs on the fused kernels of mlg_block_attention
 * (the phantoms only start each row's running softmax at maximum 0 with sum
 * phi), except fp64 with 32 channels, which takes the generic kernel; no
 * workspace. */
int mlg_block_attention_smooth(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                               int32_t channels, int32_t heads, mlg_dtype dtype,
                               const void* G_in, void* G_out, const void* Wq, const void* Wk,
                               const void* Wv, mlg_stream_t stream);

/* Bytes of device workspace that mlg_attention_stack needs: one [capacity][channels] buffer
 * for n_layers >= 2 (used only by centres the fused kernels do not cover), else 0. */
size_t mlg_attention_stack_workspace_bytes(int64_t capacity, int32_t channels, int32_t n_layers,
                                           mlg_dtype dtype);

/* n_layers stacked block-dense attention layers, G^{l+1} = attention(G^l) with the layer-l
 * weights; G^0 = G_in, the last layer's output in G_out.  Same per-layer definition as
 * mlg_block_attention.  A centre's output rows depend only on its own input rows, so the
 * layers of a centre run back to back on chip (one fused launch for the supported shapes)
 * and intermediate layers never reach global memory.
 *   W   HOST array of 3 * n_layers device pointers: Wq, Wk, Wv of layer 0, then layer 1, ...
 *   ws  device workspace of ws_bytes >= mlg_attention_stack_workspace_bytes() (may be NULL
 *       when that is 0) */
int mlg_attention_stack(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                        int32_t channels, int32_t heads, int32_t n_layers, mlg_dtype dtype,
                        const void* const* W, const void* G_in, void* G_out, void* ws,
                        size_t ws_bytes, mlg_stream_t stream);

/* mlg_attention_stack with the slot-occupancy softmax of
 * mlg_block_attention_smooth in every layer (the phantom count nnei_max - n of a
 * destination depends on the geometry only, so it is the same in every layer).
 * Same arguments, workspace and outputs as mlg_attention_stack. */
int mlg_attention_stack_smooth(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                               int32_t channels, int32_t heads, int32_t n_layers,
                               mlg_dtype dtype, const void* const* W, const void* G_in,
                               void* G_out, void* ws, size_t ws_bytes, mlg_stream_t stream);

/* Bytes of device workspace for mlg_forward: the build's workspace plus, for
 * n_layers >= 2, one [capacity][channels] buffer for the layer ping-pong. */
size_t mlg_forward_workspace_bytes(int64_t n_atoms, double rcut, const double box[9],
                                   const uint8_t pbc[3], int64_t capacity, int32_t channels,
                                   int32_t n_layers, mlg_dtype dtype);

/* mlg_build_csr followed by n_layers attention layers G^{l+1} = attention(G^l).
 *   W   HOST array of 3 * n_layers device pointers: Wq, Wk, Wv of layer 0, then layer 1, ...
 *   G0  device [capacity][channels]: edge features in the canonical order of the graph
 *       this call builds (the build is deterministic, so a previous build of the same
 *       coordinates gives that order)
 *   G_out device [capacity][channels], must not alias G0
 * Everything runs on `stream` without a host synchronisation (CUDA-graph capturable). */
int mlg_forward(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                int32_t channels, int32_t heads, int32_t n_layers, mlg_dtype dtype,
                const void* const* W, const void* G0, void* G_out, const mlg_csr* csr,
                void* ws, size_t ws_bytes, mlg_stream_t stream);

/* Verlet-skin reuse of the neighbour search across MD steps (DPA4 LAMMPS
 * issue, Proposed optimizations: keep the device tensors of the edge
 * construction while the neighbour list is unchanged, rebuild when the MD
 * engine's skin criterion asks for it).
 *
 * The list: every (source, shift) within rcut + skin of each destination at
 * the coordinates it was built at, as a CSR in canonical order, with no cap
 * other than 256 candidates per destination.  All members are caller-owned
 * DEVICE memory. */
typedef struct {
    mlg_csr cand;          /* candidate CSR (row_ptr [N+1], src, shift; the vec, dist and sw
                              arrays are written by its build too); capacity >= N * 256
                              always suffices */
    double* coords_ref;    /* [N][3]: the coordinates the candidates were found at */
    uint32_t* state;       /* bit 0: the list is valid.  Zero it before the first call (and
                              whenever the atoms are renumbered or the box changes) */
    int64_t* n_builds;     /* counter of list builds (diagnostics; the library adds 1 per
                              build) */
} mlg_verlet_list;

/* Bytes of device workspace that mlg_verlet_step needs; 0 for invalid arguments. */
size_t mlg_verlet_workspace_bytes(int64_t n_atoms, double rcut, double skin, const double box[9],
                                  const uint8_t pbc[3]);

/* One MD step's destination CSR through the Verlet list, all on `stream`
 * without a host synchronisation:
 *   1. a device reduction finds the largest displacement of any atom since
 *      the list was built (raw coordinates: an atom re-wrapped into the box
 *      has moved by a box length); when 2 * that >= skin, a coordinate is not
 *      finite, or bit 0 of *list->state is clear, a device word asks for a
 *      rebuild;
 *   2. the build kernels, gated on that word, rebuild the list (the regular
 *      build at rcut + skin with cap 256; types are validated there) and store
 *      the coordinates; when no rebuild is asked for they return at once;
 *   3. the refine re-evaluates every candidate at the current coordinates
 *      with the build's own operation order, keeps r < rcut, caps each
 *      destination to the nnei_max nearest by (r^2, source, shift) and writes
 *      `out` in canonical order.
 * `out` is then bit for bit what mlg_build_csr(sys, rcut, r_on, nnei_max)
 * gives at the current coordinates (pairs within rcut now were within
 * rcut + skin at the list's coordinates while no atom has moved skin / 2).
 * Resets *out->status and *out->n_truncated; the input bits of the list's
 * last build (non-finite coordinate, type range, image range) are OR-ed into
 * *out->status, and MLG_STATUS_LIST_INCOMPLETE when the list overflowed.
 *   skin      >= 0 (0 rebuilds every step)
 *   ws        >= mlg_verlet_workspace_bytes(), 256-byte aligned
 * The box and pbc must stay those the list was built with. */
int mlg_verlet_step(const mlg_system* sys, double rcut, double r_on, double skin,
                    int32_t nnei_max, const mlg_verlet_list* list, const mlg_csr* out, void* ws,
                    size_t ws_bytes, mlg_stream_t stream);

/* Size of the library's built-in scratch array for mlg_build_csr_noalloc. */
#define MLG_NOALLOC_SCRATCH_BYTES (8u << 20)

/* mlg_build_csr without a workspace argument and without any allocation.
 * No counterpart in the pages: this is a deployment aid.  Some callers cannot
 * allocate device memory: a force callback inside an MD engine that passes
 * raw device pointers but owns every allocation itself (and cannot afford the
 * device-wide synchronisation an allocation may trigger in its time step), or
 * a host plugin without an allocator of its own.  For them the scratch lives
 * in a fixed array of MLG_NOALLOC_SCRATCH_BYTES (8 MiB) in the library's own
 * device memory; every GPU that loads the library holds that array until the
 * process exits.
 *   - Same arguments, results and device status as mlg_build_csr; the CSR
 *     output buffers are still the caller's.
 *   - Returns MLG_ERR_WORKSPACE, launching nothing, when the system needs more
 *     scratch than the array holds (about 150,000 atoms for a periodic box).
 *     The array build goes without the count-to-fill key stash that
 *     mlg_build_csr_workspace_bytes() counts.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it with the current context; make that
 *     first call before any stream capture begins.  A later call under a new
 *     context of that device (after cudaDeviceReset, for instance) looks the
 *     address up again.
 *   - Every call shares the one array, and the array keeps the contents of
 *     the previous call; the build clears everything that must start at zero
 *     itself.  Two calls whose work overlaps on the GPU (different streams
 *     without ordering between them) race on the array: order them. */
int mlg_build_csr_noalloc(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                          const mlg_csr* csr, mlg_stream_t stream);

/* Number of kernel launches that one mlg_forward call with these arguments
 * issues on its stream (for accounting in benchmarks); 0 for invalid
 * arguments.  Systems small enough for the one-launch build count it as one
 * kernel; its 8-byte flag reset (a cudaMemsetAsync, not a kernel of this
 * library) is not counted, and the count assumes the driver accepts that
 * cooperative launch (if it refuses, the kernel chain of larger systems runs
 * instead). */
int mlg_forward_launch_count(int64_t n_atoms, double rcut, const double box[9],
                             const uint8_t pbc[3], int32_t nnei_max, int32_t channels,
                             int32_t heads, int32_t n_layers, mlg_dtype dtype);

/* Local attention: one query per centre (NeighborGraph issue, "Graph-native
 * alternatives", item 2: LocalAtten with queries = centres and keys = edges
 * of the destination CSR).  For centre i with n = row_ptr[i+1] - row_ptr[i]
 * edges: q = H_in[i] Wq, k_b = G_in[row_ptr[i] + b] Wk, v_b = ... Wv; per
 * head h (d = channels / heads) l_b = sw_b (q^h . k_b^h) / sqrt(d), softmax
 * over b < n, out[i]^h = sum_b P_b v_b^h; a centre without edges gets a
 * zero row.  Only the key's switch weighs the logit (the centre has no
 * distance of its own).
 *   csr      CSR from mlg_build_csr (row_ptr, sw, capacity, status used);
 *            rows must hold at most nnei_max edges (true for a CSR built
 *            with the same nnei_max); a longer row gives a zero output row and
 *            sets MLG_STATUS_ROW_TOO_LONG.
 *   H_in     device [n_centres][channels] centre features, dtype.
 *   G_in     device [E][channels] edge features in CSR order, dtype.
 *   out      device [n_centres][channels], dtype; must not alias H_in or G_in.
 *   Wq/Wk/Wv device [channels][channels] row-major (y = x W), dtype.
 * channels <= 256, channels % heads == 0, 1 <= nnei_max <= 256.  The call
 * is asynchronous on `stream`, allocates nothing and needs no workspace.
 * Returns MLG_ERR_INVALID_ARG / MLG_ERR_UNSUPPORTED for bad arguments or
 * shapes, MLG_ERR_CUDA if the launch fails; when E > capacity (status
 * MLG_STATUS_CAPACITY) it writes nothing. */
int mlg_local_attention(const mlg_csr* csr, int64_t n_centres, int32_t nnei_max,
                        int32_t channels, int32_t heads, mlg_dtype dtype, const void* H_in,
                        const void* G_in, void* out, const void* Wq, const void* Wk,
                        const void* Wv, mlg_stream_t stream);

/* Diagnostics: out[i] = 2^y[i] for i < n, by the device exponential that
 * the fp64 attention uses for its softmax weights (arguments y <= 0; -inf
 * gives 0, NaN gives NaN, y < -1000 gives 0).  y and out: device arrays of n
 * doubles.  For tests of that routine against the CUDA math library.
 * Returns MLG_ERR_INVALID_ARG for null pointers with n > 0 or n < 0,
 * MLG_ERR_CUDA if the launch fails. */
int mlg_exp2_neg(const double* y, double* out, int64_t n, mlg_stream_t stream);

/* Diagnostics: the one-launch build of a small system (mlg_build_csr's
 * arguments) with its bounded waits shortened to `polls` polls each (about
 * 0.3 us apart) and CTA 0 withholding the flag that releases the other CTAs
 * after binning.  The other CTAs' waits therefore run out: they OR
 * MLG_STATUS_TIMEOUT into *csr->status and leave; CTA 0 then gives up at the
 * grid barrier the same way.  No copy is in flight at either wait, so the
 * launch ends cleanly and the context stays usable; the CSR outputs are
 * incomplete.  For tests of the timeout path of those waits.  Returns
 * MLG_ERR_UNSUPPORTED when the system does not take the one-launch build (or
 * the driver refuses the cooperative launch), MLG_ERR_INVALID_ARG for
 * polls < 1, otherwise as mlg_build_csr. */
int mlg_build_csr_wait_test(const mlg_system* sys, double rcut, double r_on, int32_t nnei_max,
                            const mlg_csr* csr, void* ws, size_t ws_bytes, int32_t polls,
                            mlg_stream_t stream);

/* A static string naming the kernels mlg_attention_stack launches for this
 * shape (for benchmark records); "" for invalid arguments. */
const char* mlg_attention_kernels(int32_t nnei_max, int32_t channels, int32_t heads,
                                  int32_t n_layers, mlg_dtype dtype);

/* A static string naming a host status code. */
const char* mlg_status_string(int status);

/* Library version as major * 10000 + minor * 100 + patch. */
int mlg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLG_H */
