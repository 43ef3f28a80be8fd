/*
 * spa.h -- C ABI of libspa.so: SPAttention band-sparse causal attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("Making Every Head Count: Sparse Attention Without the
 * Speed-Performance Trade-off", arXiv 2511.09596, abstract and Figure 1
 * caption): the causal distance range [0, N) is split by Balanced Distance
 * Partitioning into H contiguous, non-overlapping bands of width floor(N/H)
 * or ceil(N/H), head 0 nearest; head h attends only to keys whose causal
 * distance i - j lies in its band [lo_h, hi_h).  Softmax is unchanged and only
 * runs over that permitted set ("Story of Attention -- Part 4", section 1,
 * Sparse-Attention equation).  The H heads together cover every causal pair
 * once, so a layer costs one causal O(N^2) attention.
 *
 * Conventions shared by every entry point:
 *  - Tensors q, k, v, o, dout, dq, dk, dv are bf16, layout [B][H][N][d]
 *    row-major contiguous, in DEVICE memory, 16-byte aligned; the outputs
 *    o of the forward and dq, dk, dv of the backward 32-byte aligned (they
 *    are written in 32-byte stores).  lse and the backward workspace are
 *    fp32 [B][H][N], device memory, 4-byte aligned.
 *  - The caller owns every buffer; no call allocates device memory (the
 *    one library-owned buffer is the static scratch array of
 *    spa_attn_bwd_noalloc, below).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) and never synchronise the host, except
 *    spa_device_status.
 *  - scale multiplies q.k before the softmax (1/sqrt(d) for standard
 *    attention); it must be finite and > 0, else SPA_ERR_INVAL.  Softmax
 *    statistics and accumulation are fp32.
 *  - A query row whose permitted set is empty (i < lo_h) gets o = 0 and
 *    lse = -inf; it passes no gradient.  Keys that no query reaches get
 *    dk = dv = 0.  Every element of every output is written.
 *  - Supported: d in {64, 128}; 1 <= H <= 256; 1 <= N <= 2^31 - 1;
 *    1 <= B <= 65535.
 *  - Return value: SPA_OK (0) or one of the spa_status_t codes below.  An
 *    argument error is reported before anything is launched.
 *  - Thread safety: every entry point may be called from several host
 *    threads at once.
 */
#ifndef SPA_H
#define SPA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPA_API __attribute__((visibility("default")))
#else
#define SPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum spa_status {
  SPA_OK = 0,
  SPA_ERR_INVAL = 1,       /* null pointer, bad size, bad band */
  SPA_ERR_UNSUPPORTED = 2, /* d, H or alignment outside what the kernels take */
  SPA_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
  SPA_ERR_TIMEOUT = 4      /* a device-side wait hit its time limit (see spa_device_status) */
} spa_status_t;

/* Human-readable name of a status code (static string, never NULL). */
SPA_API const char* spa_status_string(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
SPA_API int spa_version(void);

/*
 * Balanced Distance Partitioning ("Making Every Head Count", Figure 1
 * caption): lo[h] = floor(h*N/H), hi[h] = floor((h+1)*N/H), in 64-bit
 * integer arithmetic.  lo, hi: HOST arrays of H int32 entries, caller-owned.
 * Requires 1 <= H <= N <= 2^31 - 1, else SPA_ERR_INVAL.
 */
SPA_API int spa_band_bounds(int64_t N, int H, int32_t* lo, int32_t* hi);

/*
 * Forward pass.  For every (b, h, i):
 *   S_i = { j : 0 <= j <= i, lo_h <= i - j < hi_h },
 *   lse_i = log(sum_{j in S_i} exp(scale * q_i.k_j))  (natural log),
 *   o_i   = sum_{j in S_i} exp(scale * q_i.k_j - lse_i) v_j.
 * q, k, v: inputs [B][H][N][d]; o: output [B][H][N][d]; lse: output [B][H][N].
 * Bands are the Balanced Distance Partitioning ones (requires H <= N).
 */
SPA_API int spa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int64_t N, int d, float scale, void* stream);

/*
 * Same as spa_attn_fwd with explicit per-head bands: lo, hi are HOST arrays of
 * H int32 entries with 0 <= lo[h] < hi[h] <= N (bands may overlap or leave
 * gaps; lo = 0, hi = N on every head is dense causal attention per head).
 */
SPA_API int spa_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int H, int64_t N, int d, float scale,
                    const int32_t* lo, const int32_t* hi, void* stream);

/*
 * Forward that merges: o and lse hold, on entry, the output and lse of a
 * softmax over another set of keys per row (for example spa_attn_fwd_ex on
 * other bands), disjoint from the bands given here; on return they hold the
 * softmax over the union of the two sets:
 *   L = log(e^lse + e^lse_here),  o = e^(lse - L) o + e^(lse_here - L) o_here,
 * computed per row in the kernel's epilogue.  Rows these bands leave empty
 * keep o and lse as they were.  Same arguments and rules as spa_attn_fwd_ex
 * (lo, hi both NULL for the Balanced Distance Partitioning bands).
 */
SPA_API int spa_attn_fwd_merge(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int64_t N, int d, float scale,
                               const int32_t* lo, const int32_t* hi, void* stream);

/* Bytes of device workspace that spa_attn_bwd needs: 4 * B * H * N (the fp32
 * row sums D_i = sum_c dout_ic * o_ic).  Returns 0 on bad sizes. */
SPA_API size_t spa_attn_bwd_workspace_bytes(int B, int H, int64_t N);

/*
 * Backward pass: gradients of L = sum(o * dout) with respect to q, k, v.
 * The pages give no backward; it is the derivative of the forward above:
 *   P_ij  = exp(scale * q_i.k_j - lse_i)   (j in S_i),
 *   D_i   = sum_c dout_ic o_ic,
 *   dS_ij = P_ij (dout_i.v_j - D_i),
 *   dq_i  = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j  = sum_i P_ij dout_i.
 * Inputs q, k, v, o (forward output), dout, lse (forward output); outputs dq,
 * dk, dv [B][H][N][d].  workspace: device buffer of at least
 * spa_attn_bwd_workspace_bytes(B, H, N) bytes, caller-owned, contents
 * overwritten.  dq, dk, dv must not alias any input.
 */
SPA_API int spa_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                 const void* dout, const float* lse, void* dq, void* dk, void* dv,
                 void* workspace, int B, int H, int64_t N, int d, float scale,
                 void* stream);

/* Backward with explicit per-head bands (same rules as spa_attn_fwd_ex). */
SPA_API int spa_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv,
                    void* workspace, int B, int H, int64_t N, int d, float scale,
                    const int32_t* lo, const int32_t* hi, void* stream);

/*
 * Backward in one pass over the key tiles: the same gradients as
 * spa_attn_bwd (the derivative written above), with S and dP computed once
 * per tile pair instead of once in each of two passes.  dk and dv are
 * accumulated per key tile as in spa_attn_bwd; dq is produced per (key tile,
 * query tile) pair and summed over the key tiles in an fp32 buffer by
 * reduction operations, then rounded to bf16 once.  Because those sums
 * arrive in no fixed order, dq may differ in its last bits from one call to
 * the next (dk and dv are bit-reproducible); spa_attn_bwd is the
 * deterministic backward.
 *   workspace: DEVICE buffer of spa_attn_bwd_fused_workspace_bytes(B, H, N, d)
 *              bytes, 256-byte aligned, caller-owned, contents overwritten
 *              (D and the fp32 sums; nothing in it needs to be initialised)
 *   lo, hi:    HOST band arrays (rules of spa_attn_fwd_ex) or both NULL for
 *              the Balanced Distance Partitioning bands
 * Other arguments, layouts and errors as spa_attn_bwd; dk and dv must be
 * 32-byte aligned and dq 16-byte aligned.
 */
SPA_API size_t spa_attn_bwd_fused_workspace_bytes(int B, int H, int64_t N, int d);
SPA_API int spa_attn_bwd_fused(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               void* workspace, int B, int H, int64_t N, int d, float scale,
                               const int32_t* lo, const int32_t* hi, void* stream);

/*
 * The three launches of spa_attn_bwd_fused, callable one at a time (to time
 * each, or to let other work run between them); `steps` is a bit mask, and
 * the three bits together are spa_attn_bwd_fused:
 *   1  D_i = sum_c dout_ic o_ic into the workspace and the fp32 dq sums set
 *      to zero, for every row of the query tiles some band reaches; dq = 0 on
 *      the rows before them;
 *   2  the pass over the key tiles: dk and dv written, dq sums added to;
 *   4  dq = bf16(scale * sums) on the rows of the reached query tiles.
 * Each step needs the ones before it to have run on the same workspace.  A
 * mask outside [1, 7] is SPA_ERR_INVAL.
 */
SPA_API int spa_attn_bwd_fused_steps(const void* q, const void* k, const void* v, const void* o,
                                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                     void* workspace, int B, int H, int64_t N, int d, float scale,
                                     const int32_t* lo, const int32_t* hi, void* stream, int steps);

/*
 * Backward that stores dS: the same gradients as spa_attn_bwd (the
 * derivative written above), bit-reproducible, with S and dP computed once per
 * tile pair.  The dK/dV pass, which forms each 128 x 128 tile pair's dS^T in
 * bf16 for its dK product, also writes it to the workspace.  The dQ pass then
 * computes dq_i = scale sum_j dS_ij k_j from the stored tiles and k alone,
 * instead of computing S and dP again.  It runs three kernels: D (for the
 * 128-row query tiles the bands reach), dK/dV, dQ.
 *   workspace: DEVICE buffer of spa_attn_bwd_stored_workspace_bytes(B, H, N,
 *              d, lo, hi) bytes, 256-byte aligned, caller-owned, contents
 *              overwritten (D, then the dS^T tiles; nothing in it needs to
 *              be initialised).  Its size is about 2 bytes per causal pair
 *              of every (b, h), plus padding: 1.25 GB for B1 H32 N32768 with
 *              the Balanced Distance Partitioning bands.  The size function
 *              returns 0 on bad sizes or bands, or past the tile limit below.
 *   dq, dk, dv: 32-byte aligned.  lo/hi: HOST band arrays, or both NULL for
 *              the Balanced Distance Partitioning bands.
 * Other tensors and rules as spa_attn_bwd.  A tile count past 2^31 - 1 is
 * SPA_ERR_UNSUPPORTED.
 */
SPA_API size_t spa_attn_bwd_stored_workspace_bytes(int B, int H, int64_t N, int d, const int32_t* lo,
                                                   const int32_t* hi);
SPA_API int spa_attn_bwd_stored(const void* q, const void* k, const void* v, const void* o,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                void* workspace, int B, int H, int64_t N, int d, float scale,
                                const int32_t* lo, const int32_t* hi, void* stream);
/*
 * The same backward one launch at a time, for timing each kernel: `steps` is
 * a bitmask, 1 = D, 2 = the dK/dV pass (dk, dv and the dS^T tiles), 4 = the
 * dQ pass from the stored tiles; spa_attn_bwd_stored runs 7.  Each step needs
 * the ones before it to have run on the same workspace.  A mask outside
 * [1, 7] is SPA_ERR_INVAL.
 */
SPA_API int spa_attn_bwd_stored_steps(const void* q, const void* k, const void* v, const void* o,
                                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                      void* workspace, int B, int H, int64_t N, int d, float scale,
                                      const int32_t* lo, const int32_t* hi, void* stream, int steps);

/*
 * The three steps spa_attn_bwd runs, callable one by one (for example to run
 * the dk/dv and dq passes on two streams once the first step is done).  Same
 * tensors and rules as spa_attn_bwd; lo/hi are HOST band arrays or both NULL
 * for the Balanced Distance Partitioning bands.
 *  1. spa_attn_bwd_preprocess: workspace[b,h,i] = D_i = sum_c dout_ic o_ic.
 *  2. spa_attn_bwd_dkdv: dk, dv from q, k, v, dout, lse and D (one CTA per key
 *     tile, walking the query tiles its band reaches).
 *  3. spa_attn_bwd_dq:   dq from q, k, v, dout, lse and D (one CTA per query
 *     tile, walking the same key strip as the forward).
 * Steps 2 and 3 only read the workspace and may run concurrently.
 *
 * spa_attn_bwd_dq_delta is steps 1 and 3 in one pass, the way spa_attn_bwd
 * runs them: the dq pass stages each 128-row block of o next to dout and
 * forms D there (fp32 sums of bf16 products, the same definition as step 1),
 * writes it to the workspace for every row of the query blocks the band
 * reaches, and computes dq.  spa_attn_bwd_dkdv run after it on the same
 * workspace completes the backward.
 */
SPA_API int spa_attn_bwd_preprocess(const void* o, const void* dout, void* workspace, int B, int H,
                                    int64_t N, int d, void* stream);
SPA_API int spa_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout,
                              const float* lse, const void* workspace, void* dk, void* dv, int B,
                              int H, int64_t N, int d, float scale, const int32_t* lo,
                              const int32_t* hi, void* stream);
SPA_API int spa_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dout,
                            const float* lse, const void* workspace, void* dq, int B, int H,
                            int64_t N, int d, float scale, const int32_t* lo, const int32_t* hi,
                            void* stream);
/*
 * spa_attn_bwd_dkdv_add and spa_attn_bwd_dq_add: the dk/dv and dq passes,
 * adding their gradients to what dk, dv (dq) hold -- each element read, the
 * pass's fp32 value added, the sum rounded once to bf16 -- instead of
 * overwriting them; rows the pass does not reach (keys no query of the band
 * reaches, queries before the band) are left as they are.  For summing the
 * passes of several disjoint bands that share one lse and D (the band plus
 * shared window calls below use them for their second part).  Same
 * arguments and errors as spa_attn_bwd_dkdv / spa_attn_bwd_dq.
 */
SPA_API int spa_attn_bwd_dkdv_add(const void* q, const void* k, const void* v, const void* dout,
                                  const float* lse, const void* workspace, void* dk, void* dv, int B,
                                  int H, int64_t N, int d, float scale, const int32_t* lo,
                                  const int32_t* hi, void* stream);
SPA_API int spa_attn_bwd_dq_add(const void* q, const void* k, const void* v, const void* dout,
                                const float* lse, const void* workspace, void* dq, int B, int H,
                                int64_t N, int d, float scale, const int32_t* lo, const int32_t* hi,
                                void* stream);
SPA_API int spa_attn_bwd_dq_delta(const void* q, const void* k, const void* v, const void* o,
                                  const void* dout, const float* lse, void* workspace, void* dq,
                                  int B, int H, int64_t N, int d, float scale, const int32_t* lo,
                                  const int32_t* hi, void* stream);

/*
 * Backward pass that allocates nothing and takes no workspace argument.
 * The paper has no counterpart: this entry point exists for callers that
 * cannot call cudaMalloc -- for example a plugin running inside a host
 * framework that owns all device memory through its own pool allocator (a
 * raw cudaMalloc behind its back would escape its budget), or a caller that
 * must not risk the device-wide synchronisation cudaMalloc/cudaFree may
 * cause.  Same inputs, outputs and results as spa_attn_bwd with the Balanced
 * Distance Partitioning bands.
 *  - Scratch: the row sums D live in a library-owned, file-scope device array
 *    of SPA_NOALLOC_MAX_ROWS floats (4 MiB), held by every GPU that loads the
 *    library until the process exits.  B * H * N above SPA_NOALLOC_MAX_ROWS is
 *    rejected with SPA_ERR_UNSUPPORTED before anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it with the
 *    id of the context it belongs to; make that first call before any stream
 *    capture.  A device reset (cudaDeviceReset) destroys the context and the
 *    array with it: the first call in the new context looks the address up
 *    again, and that call too belongs before any capture.
 *  - All calls share the one array and it keeps the last call's contents
 *    (nothing in it needs to start at zero: each call rewrites the rows it
 *    uses before reading them).  Calls whose work overlaps on the GPU -- two
 *    streams, or two host threads -- race on it; serialise them.
 */
#define SPA_NOALLOC_MAX_ROWS (1 << 20)
SPA_API int spa_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                 const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                 int B, int H, int64_t N, int d, float scale, void* stream);

/*
 * Decode step: one new token per sequence.  Each head attends only to its
 * own band of causal distances ("Making Every Head Count", abstract and
 * Figure 1 caption), so the query at position t of head h reads just the
 * cached keys j with lo_h <= t - j < hi_h -- at most the band's width,
 * whatever t is -- with the softmax over that set ("Story of Attention --
 * Part 4", section 1, the Sparse-Attention equation).
 *   q:         DEVICE bf16 [B][H][d], the new tokens' queries
 *   k, v:      DEVICE bf16 [B][H][N][d], the key/value cache (row j holds
 *              position j; only the band's rows are read)
 *   pos:       DEVICE int32 [B], the position of each sequence's new token;
 *              a position outside [0, N) gives that sequence o = 0, lse = -inf
 *   o:         DEVICE bf16 [B][H][d]
 *   lse:       DEVICE fp32 [B][H], natural log; -inf when the band holds no
 *              key yet (pos < lo_h), with o = 0
 *   workspace: DEVICE buffer of spa_attn_decode_workspace_bytes(B, H, N, d,
 *              lo, hi) bytes, caller-owned, overwritten
 *   lo, hi:    HOST band arrays (rules of spa_attn_fwd_ex) or both NULL for
 *              the Balanced Distance Partitioning bands of length N
 * Equals row pos[b] of spa_attn_fwd on the sequence whose row pos[b] holds q.
 * Two launches (a split over 256-key chunks, then their merge), asynchronous
 * on `stream`; nothing is allocated.  SPA_ERR_INVAL for null pointers, bad
 * bands or a scale that is not finite and > 0; SPA_ERR_UNSUPPORTED for
 * d not in {64, 128}, H > 256, B > 65535 or misaligned buffers (16 bytes for
 * q, k, v, o; 4 for pos, lse, workspace).  The workspace size is 0 for
 * arguments the call would reject.
 */
SPA_API size_t spa_attn_decode_workspace_bytes(int B, int H, int64_t N, int d, const int32_t* lo,
                                               const int32_t* hi);
SPA_API int spa_attn_decode(const void* q, const void* k, const void* v, const int32_t* pos, void* o,
                            float* lse, void* workspace, int B, int H, int64_t N, int d, float scale,
                            const int32_t* lo, const int32_t* hi, void* stream);

/*
 * Band plus a local window shared by every head.  "Making Every Head Count",
 * Figure 2(b), presents its EBALL ablation as the exclusive bands with local
 * sharing taken out; the pages never define the shared part, and the reading
 * built here gives every head h the permitted set
 *   S_i^h = { j <= i : i - j < window  or  lo_h <= i - j < hi_h },
 * with the softmax over S_i^h as in spa_attn_fwd.  Every row attends at least
 * to itself (window >= 1), so no row is empty.
 *   window:    1 <= window <= N, the shared distances [0, window)
 *   lo, hi:    HOST band arrays (rules of spa_attn_fwd_ex) or both NULL for the
 *              Balanced Distance Partitioning bands
 *   workspace: (backward only) DEVICE buffer of
 *              spa_attn_union_workspace_bytes(B, H, N, d) bytes for the row
 *              sums D, 32-byte aligned, caller-owned, overwritten
 * Other arguments, layouts and alignment as in spa_attn_fwd / spa_attn_bwd.
 * Each head's set is split into two disjoint, non-empty distance intervals
 * and the band kernels run once per part: the forward of the second part
 * merges into the first's o and lse (spa_attn_fwd_merge), the backward runs
 * the dQ and dK/dV passes of each part with the joint lse and D, the second
 * part's passes adding their gradients to the first's in their epilogues
 * (spa_attn_bwd_dq_add, spa_attn_bwd_dkdv_add): two launches forward, four
 * backward.  lse and o passed to
 * spa_attn_bwd_union must come from spa_attn_fwd_union.
 * SPA_ERR_INVAL for a window outside [1, N], bad bands, null pointers or a
 * bad scale; SPA_ERR_UNSUPPORTED where spa_attn_fwd / spa_attn_bwd would
 * return it, for a misaligned workspace, or when some head's set is a single
 * distance (it cannot be split).  The workspace size is 0 for shapes the
 * calls reject.
 */
SPA_API size_t spa_attn_union_workspace_bytes(int B, int H, int64_t N, int d);
/* The split the two union calls use, on the host: head h's set is the
 * distances [a1[h], b1[h]) u [a2[h], b2[h]), disjoint and non-empty -- the
 * window and the band when window < lo_h, else the two halves of
 * [0, max(window, hi_h)).  a1, b1, a2, b2: HOST arrays of H int32.  Same
 * argument rules and errors as spa_attn_fwd_union's window and bands. */
SPA_API int spa_union_parts(int64_t N, int H, int64_t window, const int32_t* lo, const int32_t* hi,
                            int32_t* a1, int32_t* b1, int32_t* a2, int32_t* b2);
/* Two steps for composing bands by hand from outputs computed into separate
 * buffers (the union calls themselves merge and add inside the kernels'
 * epilogues, spa_attn_fwd_merge and the _add passes):
 *  spa_attn_union_merge: o, lse (part 1, DEVICE, overwritten) and o2, lse2
 *    (part 2, DEVICE) -> softmax over the union of the two disjoint sets:
 *    L = log(e^lse + e^lse2), o = e^(lse - L) o + e^(lse2 - L) o2, lse = L
 *    (a row empty in both parts stays o = 0, lse = -inf).
 *  spa_attn_union_add_grads: dq += dq2, dk += dk2, dv += dv2 (DEVICE bf16
 *    [B][H][N][d], summed in fp32 and rounded once), for gradients of two
 *    parts computed into separate buffers.
 * Tensors 16-byte aligned (lse, lse2: 4).  SPA_ERR_INVAL for null pointers or
 * bad sizes, SPA_ERR_UNSUPPORTED as for spa_attn_fwd. */
SPA_API int spa_attn_union_merge(void* o, float* lse, const void* o2, const float* lse2, int B, int H,
                                 int64_t N, int d, void* stream);
SPA_API int spa_attn_union_add_grads(void* dq, void* dk, void* dv, const void* dq2, const void* dk2,
                                     const void* dv2, int B, int H, int64_t N, int d, void* stream);
SPA_API int spa_attn_fwd_union(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int64_t N, int d, float scale, int64_t window,
                               const int32_t* lo, const int32_t* hi, void* stream);
SPA_API int spa_attn_bwd_union(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, void* dq, void* dk, void* dv,
                               void* workspace, int B, int H, int64_t N, int d, float scale,
                               int64_t window, const int32_t* lo, const int32_t* hi, void* stream);

/*
 * Band tile schedule, as the kernels walk it (host evaluation of the same
 * code the device runs).  Query tile t covers rows [t*Bq, t*Bq + Bq), key
 * tile u keys [u*Bk, u*Bk + Bk); positions >= N are not permitted.
 * For each head h and query tile t (index h*nqt + t, nqt = ceil(N/Bq)):
 *   kt_begin, kt_end: first and last key tile of the diagonal strip, or
 *   kt_begin = 0, kt_end = -1 when no row of the tile has a permitted key.
 * tile_class [H][nqt][nkt] (nkt = ceil(N/Bk)): 0 = outside the strip,
 *   1 = edge (needs the per-element distance predicate), 2 = interior (every
 *   element permitted, no mask).
 * For each head h and key tile u (index h*nkt + u):
 *   qt_begin, qt_end: the query tiles the backward dk/dv pass walks for that
 *   key tile (qt_end = -1 when none).
 * All arrays are HOST memory, caller-owned; any of them may be NULL.
 * 1 <= Bq, Bk <= 4096; bands as in spa_attn_fwd_ex.
 */
SPA_API int spa_tile_schedule(int64_t N, int H, const int32_t* lo, const int32_t* hi, int Bq, int Bk,
                      int32_t* kt_begin, int32_t* kt_end, uint8_t* tile_class,
                      int32_t* qt_begin, int32_t* qt_end);

/*
 * The tile_class matrix of spa_tile_schedule computed ON THE DEVICE by the
 * classification code the kernels inline.  tile_class_dev: DEVICE buffer of
 * H * nqt * nkt bytes; asynchronous on `stream`.
 */
SPA_API int spa_tile_classes_device(int64_t N, int H, const int32_t* lo, const int32_t* hi, int Bq,
                            int Bk, uint8_t* tile_class_dev, void* stream);

/*
 * Test hook for failure detection: launches one warp that waits on an
 * mbarrier nothing ever arrives on, through the same bounded wait every
 * kernel uses, with a limit of limit_ns nanoseconds (1 ns .. 1 s).  The wait
 * gives up, raises the device error word and the kernel returns normally, so
 * the next spa_device_status() reports SPA_ERR_TIMEOUT and the context stays
 * usable.  Asynchronous on `stream`.
 */
SPA_API int spa_debug_wait_timeout(int64_t limit_ns, void* stream);

/*
 * Synchronises `stream` and returns the library's device error word, then
 * clears it: SPA_OK; SPA_ERR_TIMEOUT when a kernel gave up on a wait (the
 * kernel then wrote incomplete outputs and released its tensor memory); or
 * SPA_ERR_UNSUPPORTED when a kernel found its dynamic shared memory too
 * small for its tiles after aligning the base to 1024 bytes (it returned
 * without writing its outputs).
 */
SPA_API int spa_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPA_H */
