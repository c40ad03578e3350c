/*
 * ws.h -- C ABI of the performer unit-step library (libws.so).
 *
 * The library implements, on one B200 (sm_100a), the per-unit denoising step of
 * the Wan-Streamer v0.2 performer as described on the pages about that report:
 *
 *   - a preallocated K/V history cache into which each incoming thinker K/V
 *     slice is written in place ("Wan-Streamer v0.2：更高分辨率，相同延迟",
 *     paper.rainbus.top, section 前置知识, entry K/V缓存预分片; "Technical
 *     Summary: Wan-Streamer v0.2", gist.science, section Methodology, item 2,
 *     K/V Handling), and into which the generated latents are committed after
 *     each unit (paper.rainbus.top, section 核心方法);
 *   - block-causal attention at the granularity of one 160 ms streaming unit:
 *     a token sees all tokens of its own unit and of earlier units, none of a
 *     later one ("通义实验室发布 Wan-Streamer v0.2…", remio.ai, section
 *     为什么端到端模型对级联式 AI 智能体构成挑战), using cached K/V instead of
 *     recomputing the history (remio.ai, section 思考者与执行者的分工掩盖了更高分辨率的成本);
 *   - the flow-matching Euler update of the latent, x <- x + dt*v
 *     (paper.rainbus.top, section 核心方法, flow-matching latent generation).
 *
 * Every call runs on one GPU.  The pages split the performer across GPUs with
 * Ulysses context parallelism; here that split is a layer above this ABI
 * (per-rank caches holding a head shard each, exchanges over torch.distributed).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - bf16 tensors are passed as pointers to their 16-bit patterns (uint16_t).
 *  - Every tensor pointer is DEVICE memory owned by the caller, 16-byte aligned
 *    (else WS_ERR_ALIGN), dense row-major in the layout stated at each call.
 *  - Calls are asynchronous and ordered on the given stream (NULL = the legacy
 *    default stream).  None synchronises, except ws_sync and ws_cache_destroy.
 *    The caller keeps inputs alive and unmodified until the work on the stream
 *    has consumed them.
 *  - Argument errors are detected on the host before any launch and leave all
 *    state unchanged.  A CUDA launch error returns WS_ERR_CUDA.  Errors found by
 *    a kernel (a bounded wait that ran out) are stored in the cache's device
 *    status word and reported by the next ws_sync.
 *  - The library owns the cache memory, its slot table, the split-K workspace and
 *    the status word.  A cache belongs to the device that was current when it was
 *    created; calls on it must be made with that device current.
 *
 * Shapes: L = n_layers, H = n_heads, D = head_dim (64 or 128),
 * Nq = n_video + n_audio (latent tokens generated per unit), Nc = n_cond
 * (thinker conditioning tokens per unit), T = Nc + Nq (tokens per unit slot),
 * U = history_units, C = U + 1 (ring slots).
 */
#ifndef WS_H
#define WS_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every call. */
enum {
  WS_OK = 0,
  WS_ERR_ARG = -1,             /* bad pointer, size, layer, segment or configuration */
  WS_ERR_ALIGN = -2,           /* a tensor pointer is not 16-byte aligned */
  WS_ERR_OOM = -3,             /* device allocation failed in ws_cache_create */
  WS_ERR_UNIT_ORDER = -4,      /* unit older than the newest conditioned unit */
  WS_ERR_EVICTED = -5,         /* the unit's slot has been reused by a newer unit */
  WS_ERR_NOT_READY = -6,       /* the unit (or its latent segment) was never written */
  WS_ERR_CUDA = -7,            /* a CUDA runtime call or launch failed */
  WS_ERR_DEVICE_TIMEOUT = -8,  /* a kernel's bounded wait ran out (reported by ws_sync) */
  WS_ERR_UNSUPPORTED = -9,     /* valid request outside what this build supports (e.g. D not 64/128) */
  WS_ERR_DEVICE_CHECK = -10    /* a device-side index check failed (libws_debug.so only; ws_sync) */
};

/* Segments of a unit slot: the thinker's conditioning tokens, then the unit's latent tokens. */
enum { WS_SEG_COND = 0, WS_SEG_LATENT = 1 };

typedef struct ws_cache ws_cache_t;   /* opaque, library-owned */

typedef struct {
  int32_t n_layers;       /* L >= 1 */
  int32_t n_heads;        /* H >= 1 */
  int32_t head_dim;       /* D: 64 or 128 */
  int32_t n_video;        /* latent video tokens per unit (>= 0) */
  int32_t n_audio;        /* latent audio tokens per unit (>= 0), unsharded, same attention set */
  int32_t n_cond;         /* thinker K/V conditioning tokens per unit (>= 0) */
  int32_t history_units;  /* U >= 0: earlier units a query can see; the ring holds C = U + 1 */
} ws_cache_config;

/*
 * ws_cache_create -- allocate and zero a K/V history cache on the current device.
 *
 * Memory: K and V planes [L][2][H][C*T][D] bf16 (plane (l, 0, h) holds K of
 * layer l, head h; (l, 1, h) holds V), token rows of slot s at [s*T, (s+1)*T):
 * first the Nc conditioning rows, then the Nq latent rows (video, then audio).
 * Also a split-K workspace and a device status word.  Nq must be >= 1; the
 * total row count C*T must fit in 2^31.  On success *out receives the handle.
 * Errors: WS_ERR_ARG (NULL pointer, bad sizes), WS_ERR_UNSUPPORTED (D),
 * WS_ERR_OOM, WS_ERR_CUDA.  The zero fill is ordered on `stream`.
 */
int ws_cache_create(ws_cache_t** out, const ws_cache_config* cfg, cudaStream_t stream);

/* Synchronise the device, free everything the handle owns, free the handle. NULL is a no-op. */
int ws_cache_destroy(ws_cache_t* h);

/*
 * ws_cache_append -- write one incoming K/V slice in place.
 *
 * seg == WS_SEG_COND: the thinker's conditioning slice of `unit`,
 *   k_slice, v_slice: [L][Nc][H][D].  Units are non-decreasing: unit < newest
 *   returns WS_ERR_UNIT_ORDER.  unit > newest starts a new unit: it claims slot
 *   unit mod C (evicting the unit that held it) and becomes the newest.
 *   unit == newest rewrites its conditioning rows.
 * seg == WS_SEG_LATENT: the commit of `unit`'s generated latents, all layers,
 *   k_slice, v_slice: [L][Nq][H][D] (committed history, paper.rainbus.top,
 *   section 核心方法).  The unit must be resident: WS_ERR_EVICTED if its slot
 *   holds a newer unit, WS_ERR_NOT_READY if its conditioning slice was never
 *   appended.
 * The copy is a bit-exact bf16 copy.  Errors: WS_ERR_ARG, WS_ERR_ALIGN, the
 * unit errors above, WS_ERR_CUDA.
 */
int ws_cache_append(ws_cache_t* h, int64_t unit, int seg,
                    const uint16_t* k_slice, const uint16_t* v_slice, cudaStream_t stream);

/*
 * ws_unit_attention -- one layer of block-causal attention for the newest unit.
 *
 * First writes k_new, v_new ([Nq][H][D], the current, still-noisy latent
 * tokens' K/V of this layer) into the unit's latent rows of `layer`; then, for
 * every head h and query row i of q ([Nq][H][D]),
 *     out[i][h] = sum_j softmax_j(q[i][h] . k_j[h] / sqrt(D)) v_j[h]
 * over the visible keys j: for every resident unit u' with
 * unit - U <= u' <= unit, its Nc conditioning rows, and its Nq latent rows of
 * this layer if they have been written (by this call for u' = unit, by an
 * earlier commit or attention call otherwise).  Within a unit the attention is
 * bidirectional (video and audio together); across units it is causal.
 * With the default kernel the write and the attention are one kernel launch
 * (the unit's own key tiles are read from k_new / v_new directly; the opt-in
 * paired kernel writes first).  q, k_new and v_new are read, like every
 * buffer argument, by work queued on `stream`, so they must stay unchanged until
 * that work has run.
 * out: [Nq][H][D] bf16 (written, not accumulated).  Arithmetic: bf16 tensor-core
 * products with fp32 accumulation, fp32 online softmax, P rounded to bf16
 * before the P.V product, RNE to bf16 at the end.
 * Errors: WS_ERR_ARG (layer, pointers), WS_ERR_ALIGN, WS_ERR_NOT_READY (unit is
 * newer than the newest conditioned unit), WS_ERR_UNIT_ORDER (unit is older
 * than the newest: the stream has moved on), WS_ERR_CUDA.
 */
int ws_unit_attention(ws_cache_t* h, int layer, int64_t unit,
                      const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                      uint16_t* out, cudaStream_t stream);

/*
 * ws_prefill_attention -- block-causal attention of several consecutive query
 * units at once (a prompt prefill or any full recomputation of a stretch of
 * units), in one launch.  Query unit j = unit_first + j uses rows
 * [j*Nq, (j+1)*Nq) of q, k_new, v_new and out ([n_units][Nq][H][D]); like
 * ws_unit_attention it first writes each unit's k_new, v_new into its latent
 * rows of `layer`, then every row of unit j sees the tokens of the resident
 * units j - U .. j, never those of a later unit (block-causal across units,
 * remio.ai, section 为什么端到端模型对级联式 AI 智能体构成挑战).  Key tiles of
 * units outside a query unit's window are never loaded.  All query units must
 * have their conditioning slice appended, the last one being the newest unit;
 * 1 <= n_units <= 64.
 * Errors: as ws_unit_attention; WS_ERR_NOT_READY / WS_ERR_EVICTED if a query
 * unit is not resident; WS_ERR_EVICTED if a unit inside some query window has
 * been overwritten (n_units larger than the ring allows); WS_ERR_UNSUPPORTED
 * for n_units > 64.
 */
int ws_prefill_attention(ws_cache_t* h, int layer, int64_t unit_first, int32_t n_units,
                         const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                         uint16_t* out, cudaStream_t stream);

/*
 * ws_flow_step -- fused flow-matching Euler update, in place:
 *     x[i] <- RN_bf16( fl64( x[i] + fl64(dt * v[i]) ) ),   0 <= i < n
 * (paper.rainbus.top, section 核心方法).  dt*v is exact in fp64; the sum is
 * rounded once to fp64 and once to bf16, round-to-nearest-even; every NaN
 * result is stored as 0x7FC0.  x and v: n bf16 elements, 16-byte aligned,
 * x and v must not overlap unless x == v.  n == 0 is a no-op.
 * Errors: WS_ERR_ARG (NULL with n > 0, n < 0), WS_ERR_ALIGN, WS_ERR_CUDA.
 */
int ws_flow_step(uint16_t* x, const uint16_t* v, float dt, int64_t n, cudaStream_t stream);

/*
 * ws_cache_read -- copy one segment of one resident unit and layer out of the
 * cache (a bit-exact readback for tests and checkpoints).  k_out, v_out:
 * [Nc][H][D] for WS_SEG_COND, [Nq][H][D] for WS_SEG_LATENT.
 * Errors: WS_ERR_ARG, WS_ERR_ALIGN, WS_ERR_EVICTED, WS_ERR_NOT_READY (never
 * appended, or the latent rows of that layer were never written), WS_ERR_CUDA.
 */
int ws_cache_read(ws_cache_t* h, int layer, int64_t unit, int seg,
                  uint16_t* k_out, uint16_t* v_out, cudaStream_t stream);

/* Copy the slot table (C entries: the unit held by each slot, -1 = empty) to host memory. */
int ws_cache_slot_table(const ws_cache_t* h, int64_t* slot_unit_host);

/* Sizes derived from the configuration. */
typedef struct {
  int32_t slots;               /* C */
  int32_t tokens_per_unit;     /* T */
  int32_t n_query;             /* Nq */
  int64_t newest_unit;         /* -1 before the first append */
  uint64_t cache_bytes;        /* K and V planes */
  uint64_t workspace_bytes;    /* split-K partials */
  int32_t n_sessions;          /* 1 for ws_cache_create */
} ws_cache_info;

int ws_cache_get_info(const ws_cache_t* h, ws_cache_info* info);

/*
 * ws_cache_set_splits -- work decomposition of each attention call.  The
 * attention kernel is persistent: one lane of CTAs per pair of 128-row query
 * tiles; the CTAs of a lane share out its (head, key tile) iterations in equal
 * contiguous ranges.  A (head, query pair) item whose range is cut between
 * CTAs is written as fp32 partials and merged: by the last CTA to finish a
 * share of it, in the same launch, when every CTA runs at least 64 iterations,
 * else by a second, short kernel.  n_split = CTAs per lane:
 * 0 = automatic (one CTA per SM over all lanes), 1..1024 forces that count
 * (reduced if the partials would not fit the workspace).
 */
int ws_cache_set_splits(ws_cache_t* h, int n_split);

/*
 * ws_sync -- synchronise `stream`, then read and clear the device status word.
 * Returns WS_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait since the
 * last ws_sync, WS_ERR_DEVICE_CHECK if a device-side index check failed (only
 * the checked build, libws_debug.so, has these checks: every computed cache row,
 * output row, partial slot and merge counter is tested against its buffer's
 * bounds, and a failing access is skipped instead of made), WS_ERR_CUDA on a
 * CUDA error, else WS_OK.
 */
int ws_sync(ws_cache_t* h, cudaStream_t stream);

/* Static, human-readable text of a status code. */
const char* ws_status_string(int status);

/*
 * Launch accounting of the attention path, for benchmarks.  While enabled, the
 * library records a CUDA event pair around each attention kernel and each
 * latent write and merge kernel (combine_*) it launches (on the caller's
 * stream); calls that merge inside the attention kernel launch no merge.
 * ws_profile_read synchronises those events and returns the totals since the
 * last reset.
 */
typedef struct {
  int64_t attention_launches;
  double attention_ms;         /* sum of event-timed durations */
  int64_t combine_launches;
  double combine_ms;
  int64_t latent_write_launches;
  double latent_write_ms;
  int32_t last_n_split;        /* CTAs per query-pair lane of the last attention call */
  int32_t last_ctas;           /* CTAs of the last attention launch */
  int64_t last_keys;           /* visible keys of the last attention call */
  int32_t last_kernel;         /* kernel of the last attention launch: 1 single-SM, 2 pairs of SMs */
} ws_profile;

int ws_profile_enable(ws_cache_t* h, int enable);   /* enabling resets the totals */
int ws_profile_read(ws_cache_t* h, ws_profile* out);

/*
 * ws_debug_inject_stall -- test hook for the failure-detection path.  While
 * tile >= 0, every attention kernel of this cache leaves out the V load of its
 * CTA-local key tile `tile`, so each CTA's bounded wait for it runs out: the
 * kernel leaves its loops, drains its copies, frees TMEM and stores
 * WS_ERR_DEVICE_TIMEOUT for ws_sync (the output of that call is undefined).
 * tile = -1 turns it off.  The wait bound is 2 s, or WS_WAIT_TIMEOUT_MS (read
 * when the cache is created).  With h = NULL the hook applies to the calls of
 * ws_attention_noalloc instead (process-wide; their bound is read at each call),
 * whose status ws_attention_noalloc_sync reports.
 */
int ws_debug_inject_stall(ws_cache_t* h, int tile);

/*
 * ws_plan_visible -- host-only planning step of ws_unit_attention, exposed for
 * tests: the key rows of one (layer, head) plane that a query of `unit` sees,
 * as maximal runs of consecutive rows [row_begin[i], row_begin[i] + rows[i]).
 * slot_unit: C entries as from ws_cache_slot_table; latent_ready: C*L bytes,
 * entry [s*L + l] nonzero when slot s holds latent rows of layer l (the query
 * unit's own latent rows count as written).  Touches no GPU.
 * Errors: WS_ERR_ARG; WS_ERR_UNSUPPORTED if more than max_runs runs are needed.
 */
int ws_plan_visible(const ws_cache_config* cfg, const int64_t* slot_unit,
                    const uint8_t* latent_ready, int layer, int64_t unit,
                    int32_t* row_begin, int32_t* rows, int32_t max_runs, int32_t* n_runs);

/*
 * ws_attention_noalloc -- block-causal attention for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is an interface
 * for callers that must not call cudaMalloc (under a framework that owns every
 * allocation and hands out only fixed buffers, or in a real-time loop that may
 * not take the allocator's locks or fail on memory halfway through a unit).
 * Such callers cannot create a ws_cache, so this call takes caller-owned K/V
 * planes and keeps its scratch (the fp32 partials of query tiles whose key
 * range is cut between CTAs, the merge counters and a status word) in a
 * file-scope device array of 48 MiB that every device loading this part of the
 * library holds until exit.
 *
 * For every head h and query row i:
 *     out[i][h] = sum_j softmax_j(q[i][h] . k_j[h] / sqrt(D)) v_j[h],  0 <= j < n_keys
 * q, out: [n_query][n_heads][head_dim]; kv: [2][n_heads][n_keys][head_dim], the K
 * planes of all heads, then the V planes (the cache's per-layer layout); all
 * caller-owned device memory, 16-byte aligned.  Same arithmetic as
 * ws_unit_attention.
 * The work runs on the current device, whose array it uses: `stream` must
 * belong to that device (else WS_ERR_ARG).  The first call on a device (and the
 * first after a device reset, which creates a new context) looks up the array's
 * device address with that device current; make it before any stream capture.
 * Calls never allocate.  All calls share the array and it keeps the last call's
 * contents: calls that overlap on the GPU race on it, so the caller serialises
 * them (one stream, or ordering between streams).  Each call clears the status
 * word and the merge counters at its start.  A kernel wait that runs out (bound
 * 2 s, or WS_WAIT_TIMEOUT_MS read at each call) leaves the output undefined and
 * sets the status word, which ws_attention_noalloc_sync reports.
 * Errors: WS_ERR_ARG, WS_ERR_ALIGN, WS_ERR_UNSUPPORTED (head_dim other than 64 or
 * 128, or partials that would not fit the 48 MiB array), WS_ERR_CUDA.
 */
int ws_attention_noalloc(const uint16_t* q, const uint16_t* kv, uint16_t* out, int32_t n_query,
                         int32_t n_keys, int32_t n_heads, int32_t head_dim, cudaStream_t stream);

/*
 * ws_attention_noalloc_sync -- waits for `stream`, then reports the status word
 * of the current device's no-alloc scratch: WS_OK, or WS_ERR_DEVICE_TIMEOUT when
 * a bounded wait of the most recent ws_attention_noalloc call on this device
 * ran out (the word is cleared after being read).  No counterpart in the
 * paper.  Allocates nothing.  Errors: WS_ERR_CUDA.
 */
int ws_attention_noalloc_sync(cudaStream_t stream);

/*
 * Unit program -- the whole device work of one streaming unit, recorded once
 * as a CUDA graph and replayed per unit.  One unit is:
 *   ws_cache_append(unit, WS_SEG_COND, cond_k, cond_v);
 *   for s in 0..S-1:  for l in 0..L-1:
 *       ws_unit_attention(l, unit, q[s][l], k_new[s][l], v_new[s][l], out[s][l]);
 *     ws_flow_step(x, vel[s], dt, n_latent);
 *   ws_cache_append(unit, WS_SEG_LATENT, commit_k, commit_v);
 * with exactly the arithmetic, the host bookkeeping and the error rules of those
 * calls.  The performer has to finish this work inside every 160 ms unit, and
 * the service overlaps the units' stages (remio.ai, section
 * 思考者与执行者的分工掩盖了更高分辨率的成本).  A graph launch replaces the unit's
 * ~490 stream launches by one, so the host can run ahead by whole units and the
 * kernels start without per-launch host gaps.
 *
 * ws_unit_io: device pointers, 16-byte aligned, owned by the caller, fixed for
 * the life of the program (the graph holds them); their contents may change
 * between launches.
 *   cond_k, cond_v      [L][Nc][H][D]   thinker's slice of the unit
 *   q, k_new, v_new     [S][L][Nq][H][D] per step and layer
 *   out                 [S][L][Nq][H][D] if out_per_call, else one [Nq][H][D]
 *                       buffer that every call overwrites
 *   x                   [n_latent]       latent, updated in place by each step
 *   vel                 [S][n_latent]    velocity of each step
 *   commit_k, commit_v  [L][Nq][H][D]   committed K/V of the unit
 */
typedef struct {
  int32_t n_steps;              /* S >= 1 */
  int32_t out_per_call;         /* 1: out is [S][L][Nq][H][D]; 0: one [Nq][H][D] buffer */
  float dt;
  int64_t n_latent;             /* >= 0 */
  const uint16_t* cond_k;
  const uint16_t* cond_v;
  const uint16_t* q;
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* out;
  uint16_t* x;
  const uint16_t* vel;
  const uint16_t* commit_k;
  const uint16_t* commit_v;
  int32_t session;              /* session of a pool (0 for a plain cache) */
} ws_unit_io;

typedef struct ws_unit_graph ws_unit_graph_t;   /* opaque */

/* Create a unit program over cache h (which must outlive it).  Records nothing
 * yet.  Errors: WS_ERR_ARG (NULL, S < 1, n_latent < 0), WS_ERR_ALIGN,
 * WS_ERR_OOM, WS_ERR_CUDA. */
int ws_unit_graph_create(ws_unit_graph_t** out, ws_cache_t* h, const ws_unit_io* io);

/*
 * ws_unit_graph_launch -- enqueue unit `unit` on `stream` as one graph launch.
 * The unit's calls are recorded on a capture stream of the program (validating
 * every argument and updating the ring bookkeeping as the direct calls would),
 * the recorded graph refreshes the program's executable graph in place
 * (cudaGraphExecUpdate; a new instantiation only when the launch structure
 * changed), and the executable graph is launched.  In steady state the
 * recorded launches differ from unit to unit only in the unit's slot rows.
 * Errors: those of the recorded calls; on an error nothing is launched and the
 * cache's bookkeeping is left as before the call.  The program's executable
 * graph is shared by its launches: calls on different streams must be ordered
 * by the caller.
 */
int ws_unit_graph_launch(ws_unit_graph_t* g, int64_t unit, cudaStream_t stream);

/* Counters of a program: launches, instantiations (structure changed) and
 * in-place updates, and the host time spent recording + updating (ms). */
typedef struct {
  int64_t launches;
  int64_t instantiations;
  int64_t updates;
  int64_t nodes;                /* kernel launches in the last recorded unit */
  double record_ms;             /* host time in capture + update, summed */
} ws_unit_graph_stats;

int ws_unit_graph_get_stats(const ws_unit_graph_t* g, ws_unit_graph_stats* out);

/* Destroy a program (synchronises its pending launches first). */
int ws_unit_graph_destroy(ws_unit_graph_t* g);

/*
 * Concurrent sessions -- several independent conversations, each with its own
 * unit ring, served by one cache (a pool) and batched into single attention
 * launches.  How many concurrent conversations one deployment can carry is the
 * open question of session economics (remio.ai, section
 * 决定 Wan-Streamer 是否重要的三个信号).
 *
 * ws_pool_create -- a cache of n_sessions rings of C = U+1 slots each, in one
 * allocation: K and V planes [L][2][H][n_sessions*C*T][D] bf16, session s owning
 * rows [s*C*T, (s+1)*C*T) of each plane.  Every session starts empty.  The
 * single-session entry points (ws_cache_append, ws_unit_attention,
 * ws_prefill_attention, ws_cache_read, ws_cache_slot_table) address session 0;
 * ws_cache_create(cfg) is ws_pool_create(cfg, 1).
 * Errors: as ws_cache_create; WS_ERR_ARG for n_sessions < 1;
 * WS_ERR_UNSUPPORTED when n_sessions*C*T >= 2^31.
 */
int ws_pool_create(ws_cache_t** out, const ws_cache_config* cfg, int32_t n_sessions, cudaStream_t stream);

/* ws_cache_append / ws_cache_read / ws_cache_slot_table on one session of a pool
 * (same contracts; WS_ERR_ARG for a session outside [0, n_sessions)). */
int ws_session_append(ws_cache_t* h, int32_t session, int64_t unit, int seg,
                      const uint16_t* k_slice, const uint16_t* v_slice, cudaStream_t stream);
int ws_session_read(ws_cache_t* h, int32_t session, int layer, int64_t unit, int seg,
                    uint16_t* k_out, uint16_t* v_out, cudaStream_t stream);
int ws_session_slot_table(const ws_cache_t* h, int32_t session, int64_t* slot_unit_host);

/* A conversation ends: its session's ring is emptied (every slot free, no
 * newest unit), so a new conversation can start in it at any unit index.  Host
 * bookkeeping only; work already enqueued is unaffected. */
int ws_session_reset(ws_cache_t* h, int32_t session);

/*
 * ws_session_attention -- one launch of block-causal attention for n query
 * units of several sessions: query unit j is unit units[j] of session
 * sessions[j] (host arrays), with its queries, current-unit K/V and output at
 * rows [j*Nq, (j+1)*Nq) of q, k_new, v_new, out ([n][Nq][H][D] bf16).  Each
 * query unit writes its k_new/v_new into its session's slot and attends over
 * its own session's window only, exactly as ws_unit_attention on that session
 * would.  The units of one session form one stretch of consecutive units in
 * the list (one unit for a streaming step, several for a prefill), the last of
 * which is that session's newest unit.  1 <= n <= 64.
 * Errors: WS_ERR_ARG (a session outside the pool, a session in two stretches
 * or a stretch of non-consecutive units, NULL, negative unit),
 * WS_ERR_ALIGN, WS_ERR_NOT_READY / WS_ERR_UNIT_ORDER / WS_ERR_EVICTED per
 * session as for ws_prefill_attention, WS_ERR_UNSUPPORTED (n > 64, or more
 * visible row runs than one launch holds), WS_ERR_CUDA.  On an error nothing
 * is launched or recorded.
 */
int ws_session_attention(ws_cache_t* h, int layer, int32_t n, const int32_t* sessions,
                         const int64_t* units, const uint16_t* q, const uint16_t* k_new,
                         const uint16_t* v_new, uint16_t* out, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WS_H */
