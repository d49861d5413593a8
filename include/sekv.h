/*
 * sekv.h - C ABI of the SeKV span-structured KV cache library (CUDA, sm_100a).
 *
 * The library implements the data-parallel hot path of SeKV (resolution-adaptive
 * KV cache with hierarchical semantic memory):
 *
 *   prefill  sekv_build_spans   surprisal boundary scan -> anchors and spans,
 *                               anchor gather, per-span weighted-mean key/value,
 *                               per-span rank-r bases (Gram + top-r eigenpairs);
 *   decode   sekv_decode_attn   per-head routing over span summaries, zoom mask,
 *                               one softmax over anchors, summaries (+log|S|) and
 *                               low-rank reconstructed tokens of zoomed spans;
 *   fetch    sekv_fetch_bases   copy the bases of zoomed spans from pinned host
 *                               memory into a device arena (cold spans).
 *
 * Sources, by page title and section:
 *   "SeKV: Resolution-Adaptive KV Cache with Hierarchical Semantic Memory" -
 *   the SeKV blog walkthrough (liuzhao09.github.io), section 2.1 Eq. (1) and the
 *   rule H_t > mu + alpha*sigma; section 2.2 Eq. (2), (3), Fig. 2, Eq. (6)-(8);
 *   section 2.3 Eq. (5), (9); and the SeKV summary page (paper.rainbus.top),
 *   workflow paragraph (Stage-2 shared softmax with the log|S| correction).
 *
 * Conventions for every entry point
 *   - All buffers are caller-owned. The library never allocates device or pinned
 *     memory and never frees anything. "device" pointers must be device memory
 *     of the current device; "host" pointers are ordinary or pinned host memory
 *     as stated; the basis home may be pinned host memory (it is read and written
 *     through unified addressing).
 *   - Element types: SEKV_F32 = float, SEKV_BF16 = bfloat16 (2 bytes). K, V, q
 *     and every stored K/V-shaped output use the descriptor's dtype; logS,
 *     inv_norm, theta, O and lse are float; counts and positions are int32;
 *     block offsets and slots are int64 element offsets.
 *   - Arrays are dense row-major in the bracket order given.
 *   - Host-side argument checks happen before any launch; on failure the call
 *     returns SEKV_ERR_INVALID_ARG / SEKV_ERR_UNSUPPORTED and launches nothing.
 *     A CUDA launch error returns SEKV_ERR_CUDA (text: sekv_last_error()).
 *     Errors found on the device (capacity overflow, a cold span in ATTEND, a
 *     bounded wait that ran out, an eigenvector solve that failed) are
 *     written to *dev_status (device int32; first error wins; 0 = ok); kernels
 *     then skip the offending work and return, they never trap.
 *   - Work is enqueued on the given stream; calls do not synchronise unless
 *     stated (sekv_fetch_bases waits on the host for the routing result).
 *   - Calls are stateless: concurrent calls on different streams with disjoint
 *     output buffers are safe.
 */
#ifndef SEKV_H_
#define SEKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SEKV_VERSION 1

typedef enum {
    SEKV_OK = 0,
    SEKV_ERR_INVALID_ARG = 1,   /* a pointer, size or enum is out of range      */
    SEKV_ERR_CAPACITY = 2,      /* a_cap, m_cap, region or arena too small        */
    SEKV_ERR_CUDA = 3,          /* a CUDA call failed (see sekv_last_error)       */
    SEKV_ERR_COLD_SPAN = 4,     /* ATTEND met a zoomed span whose bases are cold */
    SEKV_ERR_TIMEOUT = 5,       /* a bounded device wait ran out                  */
    SEKV_ERR_UNSUPPORTED = 6,   /* shape outside the compiled variants            */
    SEKV_WARN_NOT_CONVERGED = 7 /* a basis eigenvector solve failed (result kept) */
} sekv_status;

enum { SEKV_F32 = 0, SEKV_BF16 = 1 };

/* Per-token span weights for the weighted means (SeKV blog 2.2):
 * UNIFORM w_t = 1; SURPRISAL w_t = H_t / sum_S H (Eq. 2, uniform if the sum is 0);
 * SOFTMAX w_t = exp(H_t) / sum_S exp(H). */
enum { SEKV_W_UNIFORM = 0, SEKV_W_SURPRISAL = 1, SEKV_W_SOFTMAX = 2 };

/* Build steps (bit mask). SCAN and LAYOUT work per sequence, SUMMARY and BASES
 * per layer range [l0, l1). Without SCAN, LAYOUT/SUMMARY/BASES use the anchor and
 * span arrays already in the descriptor (caller-supplied segmentation). */
enum {
    SEKV_BUILD_SCAN = 1,     /* boundary rule -> a_count, anchor_pos, m_count, span_beg/end */
    SEKV_BUILD_LAYOUT = 2,   /* logS and blk_off from the spans                             */
    SEKV_BUILD_SUMMARY = 4,  /* Ka/Va gather, kbar/vbar, inv_norm                           */
    SEKV_BUILD_BASES = 8,    /* per-span A,B (keys) and C,D (values) into basis_home        */
    SEKV_BUILD_ALL = 15
};

/* Decode phases. FUSED: routing + attention over a hot cache (one pass for the
 * identity routing form; with a budget or learned routing, a routing pass and then
 * attention with its mask). ROUTE: routing only (writes zmask / route_logits).
 * ATTEND: attention reading bases through the slot table; it takes zmask, as ROUTE
 * wrote it for the same q and theta, as input; without zmask (identity form, no
 * budget) it routes again, bit-identical to ROUTE. */
enum { SEKV_FUSED = 0, SEKV_ROUTE = 1, SEKV_ATTEND = 2 };

typedef void* sekv_stream_t;   /* a cudaStream_t (NULL = legacy default stream) */
typedef void* sekv_event_t;    /* a cudaEvent_t */

/*
 * Basis storage. For each (b, l) there is a region of region_elems elements
 * (storage dtype). Span S of sequence b owns the Hkv consecutive blocks starting
 * at element blk_off[b][S] of the region, one block per kv head:
 *     block = [ A (len8 x r8) | C (len8 x r8) | B (r8 x d) | D (r8 x d) ]
 * with rS = min(rank, |S|, d), len8 = roundup(|S|, 8), r8 = roundup(rS, 8).
 * Each factor is stored 8x8-blocked: the zero-padded matrix is a row-major grid
 * of 8 x 8 tiles, every tile 64 contiguous elements (row-major inside), so that
 * element (r, c) of a matrix of padded width w8 sits at
 *     ((r / 8) * (w8 / 8) + c / 8) * 64 + (r % 8) * 8 + c % 8.
 * A tile is one 128-byte line of a bf16 factor, which the decode reads with
 * conflict-free shared-memory matrix loads; a run of token (or basis-row) groups
 * is one contiguous byte range. Padding is zero. The block size,
 * 2 len8 r8 + 2 r8 d, is a multiple of 64 elements (sekv_block_elems).
 * K_S ~ A B, V_S ~ C D (SeKV blog 2.2, Eq. (6)-(8); the rank gate, 1 unless
 * sekv_build_desc.rank_gate is given, is folded into B and D).
 */
int64_t sekv_block_elems(int32_t len, int32_t d, int32_t rank);
/* An upper bound of the region size for any segmentation with <= m_cap spans of a
 * sequence of n tokens: Hkv * (2*r8*n + m_cap*(14*r8 + 2*r8*d)) rounded up to 64,
 * r8 = min(roundup(rank, 8), d). */
int64_t sekv_basis_region_bound(int32_t n, int32_t m_cap, int32_t Hkv, int32_t d, int32_t rank);

/* ------------------------------------------------------------------------- */
/* Prefill build (SeKV blog 2.1 Eq. (1) + boundary rule; 2.2 Eq. (2), (6)-(8)) */
/* ------------------------------------------------------------------------- */
typedef struct sekv_build_desc {
    /* inputs (device) */
    const float* H;          /* [B][n] surprisal H_t = -log p(x_t | x_<t)                 */
    const void* K;           /* [B][L][Hkv][n][d] keys (all L layers; rows of [l0,l1) read) */
    const void* V;           /* [B][L][Hkv][n][d] values                                   */
    /* segmentation (device; outputs of SCAN/LAYOUT, inputs otherwise) */
    int32_t* a_count;        /* [B] anchors per sequence (boundaries + local window)       */
    int32_t* m_count;        /* [B] spans per sequence                                     */
    int32_t* anchor_pos;     /* [B][a_cap] ascending token positions of the anchors        */
    int32_t* span_beg;       /* [B][m_cap] first token of span S                           */
    int32_t* span_end;       /* [B][m_cap] one past the last token of span S               */
    float* logS;             /* [B][m_cap] log|S| (float)                                  */
    int64_t* blk_off;        /* [B][m_cap+1] element offset of span S's blocks in a region */
    double* stats;           /* optional [B][3]: mu, sigma, threshold (fp64)               */
    /* anchor and summary store (device; outputs of SUMMARY) */
    void* Ka;                /* [B][L][Hkv][a_cap][d] anchor keys                          */
    void* Va;                /* [B][L][Hkv][a_cap][d] anchor values                        */
    void* kbar;              /* [B][L][Hkv][m_cap][d] weighted-mean key per span           */
    void* vbar;              /* [B][L][Hkv][m_cap][d] weighted-mean value per span         */
    float* inv_norm;         /* [B][L][Hkv][m_cap] 1/||stored kbar|| (0 for a zero vector) */
    /* bases (output of BASES): device memory (hot) or pinned host memory (cold) */
    void* basis_home;        /* [B][L][region_elems]                                       */
    int32_t* dev_status;     /* device int32, required                                     */
    void* workspace;         /* device, sekv_build_workspace_bytes() bytes, 256-B aligned  */
    /* learned-form routing summaries (SeKV blog 2.2 Eq. (3)); optional, SUMMARY step:
     *   kbar_r[b][l][h][S] = y / ||y||_2,  y = sum_{t in S} w_t W^(l,h) K_t = (sum w) W^(l,h) kbar_S
     * for every query head h (its kv head is h / (Hq/Hkv)); the positive weight sum
     * cancels, so y is formed from the unrounded weighted mean; a zero y gives 0.  */
    const void* route_W;     /* NULL (identity routing) or [L][Hq][dr][d] W^(l,h) (storage dtype) */
    void* kbar_r;            /* [B][L][Hq][m_cap][dr] routing summaries (storage dtype, written)  */
    /* rank gate (SeKV blog 2.2 Eq. (6)): K^_S = sum_i m_i sigma_i u_i v_i^T, same for V.
     * Optional, BASES step; folded into the stored factors (row i of B / D times m_i). */
    const float* rank_gate;  /* NULL (all 1) or [B][L][Hkv][m_cap][2][rank]: the key gates then the
                                value gates of span S, component i in descending singular-value
                                order (i < rS is used)                                       */
    int64_t region_elems;    /* elements per (b, l) region of basis_home                   */
    int64_t workspace_bytes;
    double alpha;            /* boundary sensitivity: boundary iff H_t > mu + alpha*sigma   */
    int32_t B, L, Hkv, n, d, dtype;
    int32_t l0, l1;          /* layer range of SUMMARY/BASES, 0 <= l0 < l1 <= L            */
    int32_t a_cap, m_cap;    /* capacities; m_cap must be a multiple of 32                 */
    int32_t window;          /* the last `window` positions are anchors                    */
    int32_t wmode;           /* SEKV_W_*                                                    */
    int32_t rank;            /* basis rank r >= 1                                           */
    int32_t max_sweeps;      /* >= 1; kept for compatibility (the solver's steps are fixed) */
    int32_t steps;           /* SEKV_BUILD_* mask                                           */
    int32_t Hq;              /* query heads (with route_W: a multiple of Hkv, Hq/Hkv <= 8)  */
    int32_t dr;              /* routing dimension d' (with route_W: 32 or 64)               */
    int32_t reserved;
} sekv_build_desc;

size_t sekv_build_workspace_bytes(const sekv_build_desc* desc);
/* Enqueue the requested build steps on `stream`. d must be 64 or 128. BASES solves,
 * per span, key or value matrix X (|S| x d) and N = min(|S|, d), the symmetric
 * eigenproblem of the N x N Gram matrix (X X^T or X^T X, tensor cores for bf16)
 * for its top rS eigenpairs only: Householder tridiagonalisation, multisection on
 * Sturm counts, 3 steps of block inverse iteration with Gram-Schmidt, then the
 * reflectors' back-transformation (fp32). A solve that fails (a vector that vanishes
 * or a non-finite solve, none expected) raises SEKV_WARN_NOT_CONVERGED. */
sekv_status sekv_build_spans(const sekv_build_desc* desc, sekv_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Decode attention (SeKV blog 2.3 Eq. (5), (9); SeKV summary, Stage 2)      */
/* ------------------------------------------------------------------------- */
typedef struct sekv_decode_desc {
    const void* q;           /* [B][L][Hq][d] queries (storage dtype)                      */
    const int32_t* a_count;  /* [B]                                                        */
    const int32_t* m_count;  /* [B]                                                        */
    const int32_t* span_beg; /* [B][m_cap]                                                 */
    const int32_t* span_end; /* [B][m_cap]                                                 */
    const float* logS;       /* [B][m_cap]                                                 */
    const int64_t* blk_off;  /* [B][m_cap+1]                                               */
    const void* Ka;          /* [B][L][Hkv][a_cap][d]                                      */
    const void* Va;
    const void* kbar;        /* [B][L][Hkv][m_cap][d]                                      */
    const void* vbar;
    const float* inv_norm;   /* [B][L][Hkv][m_cap]                                         */
    const float* theta;      /* [L][Hq] zoom threshold in logit space, ln(tau/(1-tau))      */
    const void* arena;       /* bases: the device home [B][L][region_elems] when slot is   */
                             /* NULL, else a device arena addressed through slot           */
    const int64_t* slot;     /* NULL or [B][L][m_cap]: element offset in arena of span S's  */
                             /* Hkv blocks, -1 = cold                                      */
    float* O;                /* [B][L][Hq][d] attention output (FUSED/ATTEND)              */
    float* lse;              /* [B][L][Hq] natural-log partition (FUSED/ATTEND)            */
    uint32_t* zmask;         /* optional [B][L][Hq][m_cap/32] zoom bits (bit S%32 of word   */
                             /* S/32); required for ROUTE. Bits of spans >= m_count are 0  */
    float* route_logits;     /* optional [B][L][Hq][m_cap] routing logits l_S              */
    /* learned-form routing (SeKV blog 2.3 Eq. (5)); optional. With route_W the routing
     * logit is l_S = (W^(l,h) q_h) . kbar_r_S / sqrt(dr) + logS_S, computed by a separate
     * routing pass; zmask is then required in every phase (ROUTE writes it; FUSED
     * writes it and attends with it; ATTEND reads it as input, no re-routing). The
     * coarse entries of Stage 2 still use kbar / vbar in the key/value space.       */
    const void* route_W;     /* NULL (identity routing) or [L][Hq][dr][d] (storage dtype)  */
    const void* kbar_r;      /* [B][L][Hq][m_cap][dr] routing summaries from the build     */
    int32_t* dev_status;     /* device int32, required                                     */
    void* workspace;         /* device, sekv_decode_workspace_bytes() bytes, 256-B aligned */
    uint32_t* arrive;        /* optional [B][L][Hkv] device arrival counters, all zero before
                                the first call that gets them; every FUSED / ATTEND call leaves
                                them zero again. With them the last CTA of each (b, l, kv head)
                                to finish merges the split-K partials (no second kernel);
                                NULL = a separate merge kernel. The results are the same bits
                                either way. Calls in flight at the same time must not decode
                                the same (b, l, kv head) with the same counters.            */
    int64_t region_elems;
    int64_t workspace_bytes;
    float scale;             /* logit scale, normally 1/sqrt(d) (routing uses it too, d'=d) */
    int32_t B, L, Hq, Hkv, d, dtype;
    int32_t l0, l1;          /* layers decoded by this call                                */
    int32_t a_cap, m_cap;
    int32_t rank;
    int32_t phase;           /* SEKV_FUSED / SEKV_ROUTE / SEKV_ATTEND                       */
    int32_t nsplit;          /* CTAs per (b, l, kv head); 0 = automatic                    */
    int32_t rows_hint;       /* expected anchors + spans of a sequence (e.g. the last
                                build's counts), used by the automatic split choice;
                                0 = unknown (the choice then assumes the capacities)   */
    int32_t budget;          /* zoom budget per (b, l, query head); 0 = none. SeKV blog
                                2.3 (under Eq. (9)): when more spans pass the threshold,
                                keep them in descending alpha~ (= logit) order, equal
                                logits lower span index first. Needs zmask: ROUTE writes
                                the capped mask; ATTEND reads it as input (no re-routing);
                                FUSED routes, caps, then attends with the capped mask.
                                Without route_logits the workspace holds the logits.     */
    int32_t zoom_hint;       /* expected zoomed spans per (b, l, kv head) (e.g. from the
                                previous step); 0 = unknown. At >= 64 (and rank <= 16) a
                                decode variant that hands small spans whole to one warp
                                is used, which is faster when most spans zoom and slower
                                when few do. Results are the same either way.            */
    int32_t dr;              /* routing dimension d' with route_W (32 or 64)                */
    int32_t test_flags;      /* 0 in normal use. Bit 0 (testing the error path): the decode
                                kernels issue no copy and give every bounded wait ~4096 polls,
                                so the waits run out, *dev_status reads SEKV_ERR_TIMEOUT and the
                                kernels return with nothing in flight (O = 0, lse = -inf).   */
    int32_t static_ready;    /* 0 (default) or 1. The decode kernels are launched with
                                programmatic dependent launch: a grid may start while the
                                previous kernel on the stream finishes, and waits for it
                                before it reads its inputs. With 1 the caller guarantees
                                that no work still in flight on the stream writes the cache's
                                build outputs (a_count, m_count, Ka, Va, kbar, vbar, inv_norm,
                                logS), e.g. the stream was synchronised after the build; the
                                kernel then reads the counts and its first anchor / summary
                                tiles before that wait, so their latency overlaps the previous
                                kernel's end (a layer-by-layer decode loop). Everything else
                                (q, theta, zmask, the bases, the workspace) is still read
                                after the wait. Results are the same bits either way.     */
} sekv_decode_desc;

size_t sekv_decode_workspace_bytes(const sekv_decode_desc* desc);
/* Enqueue one decode step for layers [l0, l1) on `stream`. Hq/Hkv must be 1, 2, 4
 * or 8 and d 64 or 128. Routing logit per query head h and span S (identity form):
 *   l_S = (q_h . kbar_S) * inv_norm_S * scale + logS_S, zoom iff l_S > theta[l][h]
 * (learned form: see route_W);
 * attention over anchors (q.Ka*scale), non-zoomed spans (q.kbar*scale + logS,
 * value vbar) and the tokens of zoomed spans ((A_S (B_S q))*scale, value C_S^T-
 * weighted D_S rows), all in one softmax. */
sekv_status sekv_decode_attn(const sekv_decode_desc* desc, sekv_stream_t stream);

/*
 * Decode without a workspace. The SeKV pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory on the decode
 * path - for example a serving loop that runs inside a memory pool it does not
 * own, a plugin whose host framework forbids allocations after start-up, or code
 * that must not call cudaMalloc because cudaMalloc can synchronize the device.
 * Same contract as sekv_decode_attn, except that desc->workspace and
 * desc->workspace_bytes are ignored: the split-K partials go to one static
 * device array of SEKV_STATIC_SCRATCH_BYTES that every device which loads the
 * library holds until the process exits.
 *   - A call whose partials (sekv_decode_workspace_bytes) exceed the array is
 *     rejected with SEKV_ERR_CAPACITY and launches nothing.
 *   - No cudaMalloc, cudaFree or allocating library routine is called. The first
 *     call on a device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current) and caches it with the device's current context:
 *     make that first call before any stream capture. A call made under another
 *     context of the device (for example after cudaDeviceReset) looks the address
 *     up again, so it too should come before any capture.
 *   - Every call uses the same array, which keeps the last call's contents; each
 *     call writes all the scratch it reads, so nothing has to start at zero.
 *     Calls whose kernels can overlap on the GPU (different streams without an
 *     ordering between them) race on the array.
 */
#define SEKV_STATIC_SCRATCH_BYTES (8u << 20)
sekv_status sekv_decode_attn_static(const sekv_decode_desc* desc, sekv_stream_t stream);

/*
 * Merge decode results of disjoint parts of one logit list by log-sum-exp
 * (SeKV summary, workflow paragraph: Stage 2 is ONE softmax over every entry, so
 * results of a partition recombine exactly). Used for context-parallel decode:
 * each rank decodes the anchors and spans of its slice of the context and the
 * parts are merged after an all-gather.
 *   O_parts   [nparts][rows][d] fp32 (device), lse_parts [nparts][rows] fp32 (device)
 *   O         [rows][d] fp32 (device, written), lse [rows] fp32 (device, written)
 * A part with lse = -inf (no entries) contributes nothing; rows with no entries in
 * any part get O = 0, lse = -inf. d <= 1024, 1 <= nparts <= 64. Asynchronous on
 * `stream`; argument errors return SEKV_ERR_INVALID_ARG before any launch.
 */
sekv_status sekv_merge_partials(const float* O_parts, const float* lse_parts, int32_t nparts, int64_t rows,
                                int32_t d, float* O, float* lse, sekv_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Cold-basis fetch (SeKV summary: zoomed spans' bases fetched from the CPU;  */
/* SeKV blog Fig. 2)                                                          */
/* ------------------------------------------------------------------------- */
typedef struct sekv_fetch_desc {
    const uint32_t* zmask_dev;    /* [B][L][Hq][m_cap/32] device, written by ROUTE           */
    uint32_t* zmask_host;         /* pinned host staging of the same shape                   */
    const int32_t* m_count_host;  /* [B] host copy of m_count                                */
    const int64_t* blk_off_host;  /* [B][m_cap+1] host copy of blk_off                       */
    const int64_t* blk_off_dev;   /* optional [B][m_cap+1] device blk_off. Refill mode with it:
                                     one gather kernel reads the home through unified
                                     addressing and copies, for each (b, l, kv head), only
                                     that kv head's block of the spans its query heads zoom
                                     (the slot table still reserves a span's Hkv blocks). NULL,
                                     or a home the device cannot address: copy-engine copies
                                     of every zoomed span's Hkv blocks.                      */
    const void* home;             /* pinned host basis home [B][L][region_elems]             */
    void* arena;                  /* device arena, arena_elems elements                      */
    int64_t* slot_dev;            /* [B][L][m_cap] device slot table (written on `copy`)     */
    int64_t* slot_host;           /* pinned host mirror of the slot table                    */
    int64_t* stats;               /* optional host [5]: bytes copied, spans copied, copies,
                                     spans already resident (keep mode), spans evicted       */
    int64_t* arena_used;          /* optional host [1], written: arena elements holding bases
                                     after the call                                          */
    int64_t* arena_top;           /* optional host [1], keep mode: the end (elements) of the
                                     highest entry placed so far, read and written by every
                                     call; the caller sets it to 0 together with slot_host.
                                     Misses that fit above it are placed there without a
                                     pass over the slot table. NULL: found by that pass.     */
    int64_t* last_use;            /* keep mode: host [B][L][m_cap], the step at which each
                                     resident span was last needed; the caller sets it to -1
                                     (and slot_host to -1) once, the library keeps it        */
    sekv_event_t route_done;      /* optional (keep mode only): an event recorded right after
                                     the ROUTE call that wrote zmask_dev. The routing result is
                                     then read after this event on `copy`, so the caller may
                                     have queued later work (the previous layer's ATTEND) on
                                     `compute` and the copies overlap it. NULL: the result is
                                     read on `compute` after all work queued there.          */
    int64_t region_elems;
    int64_t arena_elems;
    int64_t step;                 /* keep mode: the caller's decode-step counter (>= 0, the
                                     same for every layer range of one step, increasing)     */
    int32_t B, L, Hq, Hkv, d, dtype;
    int32_t l0, l1, m_cap, rank;
    int32_t keep;                 /* 0: every call refills the arena with the zoomed spans of
                                     [l0, l1) (each as one copy per rectangle of consecutive
                                     spans x consecutive layers).
                                     1: the arena is a device cache across calls: spans zoomed
                                     again are not copied again. Misses are placed above the
                                     highest entry while they fit there, else first-fit in the
                                     free space below;
                                     when none fits, spans are evicted least recently used
                                     first, never one needed by this call or stamped with this
                                     step or the previous one (ATTEND calls of those steps may
                                     still be reading it; the caller must have finished every
                                     ATTEND of older steps).                                 */
    int32_t reserved;
} sekv_fetch_desc;

/* Copy the bases of every span that any query head of (b, l) zooms, for layers
 * [l0, l1), into the arena, and point the slot table at them (refill mode: -1
 * elsewhere in [l0, l1); keep mode: resident spans keep their slots, evicted ones
 * get -1). The routing result is read back first (see route_done; the host waits
 * for it); the copies and the slot-table upload go on `copy`; `done` is recorded on
 * `copy`. The caller makes `compute` wait on `done` before ATTEND. stats[2] counts
 * the copies (cudaMemcpyAsync, or cudaMemcpy2DAsync for a rectangle; with the gather
 * kernel, the kv-head blocks it moves). Returns
 * SEKV_ERR_CAPACITY, with nothing copied and both slot tables as they were, when
 * the zoomed bases that are not resident do not fit (keep mode: after every
 * allowed eviction). */
sekv_status sekv_fetch_bases(const sekv_fetch_desc* desc, sekv_stream_t compute,
                             sekv_stream_t copy, sekv_event_t done);

/* ------------------------------------------------------------------------- */
/* Zoom thresholds (SeKV blog 2.3, Eq. (9))                                   */
/* ------------------------------------------------------------------------- */
/* Eq. (9) zooms span S for a head when sigma(l_S) > tau^(l,h). The decode compares
 * in logit space instead, l_S > theta with theta = ln(tau / (1 - tau)), which is
 * the same decision without the sigmoid's saturation. This fills theta (host,
 * n floats, e.g. the [L][Hq] table that sekv_decode_desc.theta points at once it
 * is copied to the device) from tau (host, n doubles): computed in double,
 * rounded to float; tau <= 0 gives -inf (every span zooms) and tau >= 1 gives
 * +inf (none does). A NaN tau, a null pointer with n > 0, or n < 0 returns
 * SEKV_ERR_INVALID_ARG before anything is written. Synchronous, no GPU work. */
sekv_status sekv_tau_to_theta(const double* tau, float* theta, int64_t n);

/* ------------------------------------------------------------------------- */
const char* sekv_status_str(int32_t status);
const char* sekv_last_error(void);           /* thread-local detail of the last error */
size_t sekv_desc_size(int32_t which);        /* sizeof: 0 build, 1 decode, 2 fetch     */
int32_t sekv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SEKV_H_ */
