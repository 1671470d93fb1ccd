/*
 * vattn — spatiotemporal attention for video diffusion transformers and
 * streaming transformer decoders, as hand-written sm_100a (B200) kernels.
 *
 * C ABI.  Every pointer argument named q/k/v/o/ring/state/table/workspace is
 * DEVICE memory owned by the caller (allocate it with any allocator, e.g.
 * PyTorch); the library never frees caller memory.  Other pointers are host
 * memory and are read during the call only.
 *
 * Common conventions
 *  - Tensors q, k, v, o are bfloat16, contiguous, layout [B][L][H][d]
 *    (token-major, heads, then head channels): the layout a DiT QKV
 *    projection emits.  Base pointers must be 16-byte aligned.
 *  - Token n of a latent video of T x Hg x Wg tokens sits at
 *    (t, h, w) = (n / (Hg*Wg), (n / Wg) % Hg, n % Wg): row-major over the
 *    latent order B x C' x T' x H' x W' of FlashDecoder ("Preliminaries:
 *    Latent Diffusion Model", Sec. 3.1).  A "frame" is Hg*Wg consecutive
 *    tokens.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream), allocates nothing, never synchronises, and may be
 *    captured in a CUDA graph.  Arguments are checked before any launch;
 *    on an error nothing is launched and no output is touched.
 *  - Kernels bound every internal wait.  A wait that gives up records a
 *    code in a device status word; vattn_check() reports it as
 *    VATTN_ERR_TIMEOUT.
 *  - d (head dim) must be 64 or 128; H must be a multiple of Hkv.
 */
#ifndef VATTN_H_
#define VATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* vattn_stream;

typedef enum {
  VATTN_OK = 0,
  VATTN_ERR_INVALID_ARG = 1, /* a pointer, size or option is invalid          */
  VATTN_ERR_UNSUPPORTED = 2, /* valid, but not a shape the library supports   */
  VATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed             */
  VATTN_ERR_TIMEOUT = 4      /* a kernel gave up on a bounded internal wait   */
} vattn_status;

typedef enum {
  /* every query sees every key (Wan-style DiT self-attention) */
  VATTN_FULL = 0,
  /* key frame fk visible from query frame fq iff floor(fk/c) <= floor(fq/c):
     bidirectional inside a chunk of c frames, causal across chunks
     (FlashDecoder, "Effectiveness of Each Component", Sec. 4.2, the
     "full block causal attention" baseline; MobileWan chunk-wise
     autoregression) */
  VATTN_CHUNK_CAUSAL = 1,
  /* visible iff fq - window_back <= fk <= fq + window_fwd: the per-frame
     sliding window of FlashDecoder "Streaming with Rolling KV Cache"
     (Sec. 3.3) — all tokens of the query's own frame and of the window
     frames, no mask inside a frame */
  VATTN_SLIDING = 2
} vattn_mode;

/*
 * 3D rotary position embedding (FlashDecoder "Transformer Backbone Design",
 * Sec. 3.2: RoPE applied separately to the temporal and spatial axes; the
 * channel groups t / x / y of the Kaleido review; frequencies as in
 * RoFormer).  Channel pair j = (2j, 2j+1) of a head turns by angle
 * pos * theta^(-i / n_axis), where pairs [0, pairs_t) use pos = t (i = j),
 * the next pairs_h use pos = h and the last pairs_w use pos = w
 * (i = index inside the group).  pairs_t + pairs_h + pairs_w = d / 2.
 */
typedef struct {
  int Hg, Wg;                     /* spatial token grid of one frame        */
  int pairs_t, pairs_h, pairs_w;  /* channel pairs per axis                 */
  int max_pos;                    /* table rows; every t, h, w < max_pos    */
  double theta;                   /* base, e.g. 10000                       */
} vattn_rope;

/* Bytes of the cos/sin table for (rope, d): max_pos * (d/2) * 8.
   0 if the configuration is invalid. */
size_t vattn_rope_table_bytes(const vattn_rope* rope, int d);

/* Fill the caller's device table (float2 [max_pos][d/2] of (cos, sin),
   angles evaluated in double, rounded to fp32).  Build it once per
   configuration ("precomputed RoPE tables", FlashDecoder "Inference
   Optimization", Sec. 4.6). */
vattn_status vattn_rope_table_build(const vattn_rope* rope, int d, float* table,
                                    vattn_stream stream);

/*
 * Standalone 3D-RoPE of q [B][L][H][d] and k [B][L][Hkv][d] into q_out /
 * k_out (same layouts; out-of-place; q_out may not alias k).  Token n is at
 * frame t = frame_offset + n / (Hg*Wg).  fp32 rotation, bf16 round-to-
 * nearest-even results.  Either (q, q_out) or (k, k_out) may be NULL.
 */
vattn_status vattn_rope_qk(const void* q, const void* k, void* q_out, void* k_out, int B, int L,
                           int H, int Hkv, int d, const vattn_rope* rope, const float* table,
                           int frame_offset, vattn_stream stream);

/*
 * Masked softmax attention with optional fused 3D-RoPE.
 *   q [B][Lq][H][d], k/v [B][Lk][Hkv][d], o [B][Lq][H][d] (bf16).
 *   lse (nullable) fp32 [B][H][Lq]: natural log of each row's softmax
 *   denominator of scale*q.k (for combining partial attentions).
 *   Query token n is in frame q_frame_offset + n / tokens_per_frame, key
 *   token n in frame k_frame_offset + n / tokens_per_frame.  The mode picks
 *   the visible keys (see vattn_mode); tokens_per_frame is ignored by FULL
 *   unless rope is given.
 *   rope/table (both nullable): when given, q and k are rotated at their own
 *   (t, h, w) before the products; then tokens_per_frame must equal
 *   rope->Hg * rope->Wg.  The query tile is rotated inside the kernel on its
 *   shared-memory copy.  Keys: see vattn_attention_workspace_bytes.
 *   workspace (nullable, device, 16-byte aligned) of workspace_bytes: scratch
 *   for the rotated keys (unused without rope) and, when workspace_bytes
 *   reaches vattn_attention_workspace_bytes_ex, for the tail split of a FULL
 *   call (zero-filled before first use, see there).
 * o = softmax(scale * q k^T restricted to visible keys) v, computed with an
 * online softmax (fp32 statistics, fp32 accumulation, bf16 P and output).
 * Tiles with no visible key are never loaded.
 */
vattn_status vattn_attention(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Lq, int Lk, int H, int Hkv, int d, float scale,
                             vattn_mode mode, int tokens_per_frame, int chunk_frames,
                             int window_back, int window_fwd, int q_frame_offset,
                             int k_frame_offset, const vattn_rope* rope, const float* table,
                             void* workspace, size_t workspace_bytes, vattn_stream stream);

/* Bytes of workspace that let vattn_attention rotate K once per call
   (B * Lk * Hkv * d * 2 when rope is given, else 0).  With a workspace the
   call writes the rotated keys there in one HBM pass and the attention
   kernel rotates only its Q tile (once per tile); with workspace == NULL
   the kernel also rotates every K tile it loads, in shared memory. */
size_t vattn_attention_workspace_bytes(int B, int Lk, int Hkv, int d, const vattn_rope* rope);

/* Bytes of workspace that also enable the tail split of a VATTN_FULL call:
   when the call's work units (pairs of 128-row query tiles x heads x batch)
   leave a last partial wave that fills at most half the SMs of the current
   device, each unit of that wave runs as several CTAs over parts of its
   keys, merged exactly inside the kernel, so the otherwise idle SMs share
   the last wave.  The extra bytes (after the rotated keys, from a 256-byte
   boundary) hold arrival counters and fp32 partials: zero-fill the
   workspace before its first use; every call leaves the counters at zero.
   Calls sharing a workspace must not overlap on the GPU.  Equals
   vattn_attention_workspace_bytes when the split does not apply. */
size_t vattn_attention_workspace_bytes_ex(int B, int Lq, int Lk, int H, int Hkv, int d, vattn_mode mode,
                                          const vattn_rope* rope);

/*
 * Exact combination of R partial attentions of the same queries over
 * disjoint key sets (the join of Ring attention's key shards in unified
 * sequence parallelism, ReGenVC "Unified sequence parallelism", Sec. 3.5;
 * numerically equivalent to one attention over all keys up to reduction
 * order):
 *   o = sum_r e^{lse_r - M} o_r / sum_r e^{lse_r - M},  M = max_r lse_r,
 *   lse = M + ln sum_r e^{lse_r - M}.
 *   o_parts bf16 [R][B][L][H][d] and lse_parts fp32 [R][B][H][L]: the o and
 *   lse outputs of R vattn_attention calls (one per key shard), stacked;
 *   o bf16 [B][L][H][d]; lse (nullable) fp32 [B][H][L].  A part whose keys
 *   were all invisible to a row (lse = -inf) has weight 0; a row with no
 *   visible key in any part gets o = 0, lse = -inf.  1 <= R <= 64; d a
 *   multiple of 8; o_parts and o 16-byte aligned.  One HBM pass (16-byte
 *   vectors), asynchronous on `stream`.
 */
vattn_status vattn_attention_merge(const void* o_parts, const float* lse_parts, int R, void* o, float* lse, int B,
                                   int L, int H, int d, vattn_stream stream);

/*
 * Rolling KV cache of a fixed number of frames (FlashDecoder "Streaming with
 * Rolling KV Cache", Sec. 3.3; constant memory regardless of video length,
 * "Long Video Decoding", Sec. 4.3).  Storage is caller-owned device memory:
 *   k_ring, v_ring: bf16 [capacity][B][F][Hkv][d]   (raw, un-rotated K/V)
 *   frame_ids: int32 [capacity]  (frame held by each slot, -1 = empty)
 * Frame f lives in slot f mod capacity.  The handle is host metadata (with a
 * host mirror of frame_ids); it does not own the storage.
 */
typedef struct vattn_kvcache vattn_kvcache;

/* Create a handle; sets every frame_ids entry to -1 on `stream`. */
vattn_status vattn_kvcache_init(vattn_kvcache** cache, void* k_ring, void* v_ring,
                                int32_t* frame_ids, int capacity, int B, int F, int Hkv, int d,
                                vattn_stream stream);
/* Copy frame f's K and V (bf16 [B][F][Hkv][d] each) into slot f mod
   capacity and set frame_ids[slot] = f: a bit-exact 16-byte vector copy. */
vattn_status vattn_kvcache_append(vattn_kvcache* cache, const void* k, const void* v,
                                  int frame_idx, vattn_stream stream);
/*
 * One streaming step: the F query tokens of frame `frame_idx` (q bf16
 * [B][F][H][d]) attend to every token of the current frame (k_cur, v_cur,
 * [B][F][Hkv][d]) and of the cached frames frame_idx-window_back ..
 * frame_idx-1 that are present in the ring (frames before 0 do not exist).
 * No mask inside a frame; causality comes from the processing order.  Keys
 * are rotated at their own absolute frame index, queries at frame_idx.
 * window_back <= capacity.  o bf16 [B][F][H][d]; lse nullable fp32
 * [B][H][F].  Call vattn_kvcache_append for the current frame afterwards.
 */
vattn_status vattn_attention_stream(vattn_kvcache* cache, const void* q, const void* k_cur,
                                    const void* v_cur, void* o, float* lse, int H, int frame_idx,
                                    int window_back, float scale, const vattn_rope* rope,
                                    const float* table, vattn_stream stream);
/* Copy the host mirror of frame_ids (capacity entries) into host_ids. */
vattn_status vattn_kvcache_frame_ids(const vattn_kvcache* cache, int32_t* host_ids);
/* After the caller restored ring and frame_ids contents (checkpoint /
   resume), set the host mirror to host_ids (capacity entries); with a
   rotated-key ring, the restored frames' keys are rotated again on
   `stream`. */
vattn_status vattn_kvcache_restore(vattn_kvcache* cache, const int32_t* host_ids, vattn_stream stream);
/*
 * Keep a second, rotated copy of the keys so that each frame's keys are
 * rotated once, at their absolute frame index, instead of once per query
 * tile that reads them (FlashDecoder applies RoPE with precomputed tables,
 * "Inference Optimization", Sec. 4.6).  The frame tokens F must be a
 * multiple of rope->Hg * rope->Wg (F / (Hg*Wg) latent frames per cache
 * frame, see vattn_kvcache_step).  k_ring_rot: caller-owned bf16
 * [capacity + 1][B][F][Hkv][d]; frame f's rotated keys live in slot
 * f % (capacity + 1).  From then on vattn_attention_stream (which must then
 * be given the same rope and table) rotates the current frame's keys into
 * slot frame_idx % (capacity + 1), outside the window, and reads rotated keys
 * only; vattn_kvcache_append then copies the raw K and V, and also writes the
 * rotated copy in the same pass unless the last vattn_attention_stream call
 * on this cache was for the same frame with the same k pointer (those keys
 * are in place already; the caller must not change the k buffer's contents
 * between the two calls).  Frames already in the ring are rotated now, on
 * `stream`.  The raw ring stays the exact input bytes.
 */
vattn_status vattn_kvcache_enable_rope(vattn_kvcache* cache, void* k_ring_rot, const vattn_rope* rope,
                                       const float* table, vattn_stream stream);
vattn_status vattn_kvcache_destroy(vattn_kvcache* cache);

/*
 * One whole streaming step in a single launch (FlashDecoder "Streaming with
 * Rolling KV Cache", Sec. 3.3, Frame-by-Frame Processing; the fixed,
 * data-independent per-frame work that "Inference Optimization", Sec. 4.6,
 * captures in a CUDA graph): the F query tokens of frame `frame_idx` attend
 * to the current frame (k_cur, v_cur) and to the cached frames
 * frame_idx-window_back .. frame_idx-1 present in the ring, and the current
 * frame is appended: raw K and V into slot frame_idx % capacity, frame_ids
 * updated, and (with rope) its keys rotated into the rotated ring.  The
 * result equals vattn_attention_stream followed by vattn_kvcache_append.
 *  - capacity must exceed window_back: the slot written is then never one
 *    the window reads (capacity W + 1 for a window of W frames).
 *  - rope/table (both or neither): the cache must have a rotated-key ring
 *    with the same rope and table (vattn_kvcache_enable_rope).  A cache frame
 *    of F tokens holds r = F / (Hg*Wg) latent frames (r > 1: the temporal
 *    refinement layers' r_t * L_frm tokens per step, FlashDecoder
 *    "Complexity Analysis", Sec. 3.3); token n of cache frame f sits at
 *    t = r * (f - base) + n / (Hg*Wg).
 *  - window_relative = 0: base = 0 (absolute frame index).  1: base =
 *    max(0, frame_idx - window_back), positions relative to the current
 *    window ("Long Video Decoding", Sec. 4.3), so the table needs only
 *    r * (window_back + 1) frame rows however long the video; the window's
 *    earlier frames are rotated again at their new positions (one HBM pass
 *    each) before the launch.
 *  - workspace: device memory of vattn_kvcache_step_workspace_bytes(cache,
 *    H, window_back) bytes (the value depends on the current device's SM
 *    count), zero-filled before its first use; every step leaves its
 *    counters at zero.  Steps sharing a workspace must not overlap on the
 *    GPU.
 * The first CTAs of the launch copy and rotate the frame; attention CTAs
 * wait for them (a bounded wait on a counter in the workspace) only before
 * loading the current frame's rotated keys, which they reach last.  For a
 * small number of query tiles the key tiles are split across CTAs and each
 * query-tile pair's last CTA merges the partial results exactly.  When the
 * window holds no earlier frame the append runs as a separate launch first.
 * A wait that gives up records VATTN_ERR_TIMEOUT; zero the workspace again
 * before the next step after that.
 */
size_t vattn_kvcache_step_workspace_bytes(const vattn_kvcache* cache, int H, int window_back);
vattn_status vattn_kvcache_step(vattn_kvcache* cache, const void* q, const void* k_cur, const void* v_cur, void* o,
                                float* lse, int H, int frame_idx, int window_back, float scale,
                                const vattn_rope* rope, const float* table, int window_relative, void* workspace,
                                size_t workspace_bytes, vattn_stream stream);

/*
 * Hybrid chunk attention (MobileWan recurrence distillation: softmax
 * attention inside a chunk, causal linear attention across chunks through a
 * running state (s, z), feature map phi(x) = elu(x) + 1 as in Katharopoulos
 * et al.).  Tokens are cut into chunks of chunk_tokens (the last may be
 * shorter).  For query i of chunk c, with s_ij = scale * q_i . k_j:
 *   o_i = ( sum_{j in c} e^{s_ij} v_j + phi(q_i)^T S_c )
 *         / ( sum_{j in c} e^{s_ij}     + phi(q_i)^T z_c )
 * where S_c = S_in + sum_{j in chunks < c} phi(k_j) v_j^T and
 * z_c = z_in + sum phi(k_j) (phi on raw q, k; no RoPE).
 *   q/k/v/o bf16 [B][L][H][d]; S fp32 [B][H][d][d] (S[a][e]: key feature a,
 *   value channel e) and z fp32 [B][H][d] are IN/OUT: they enter as the
 *   state before token 0 and leave as the state after token L-1, so a
 *   stream of calls is the model run as an RNN.
 *   workspace: device scratch of at least vattn_hybrid_workspace_bytes().
 * Three launches: per-chunk state deltas (tcgen05 MMA), an exclusive scan
 * over chunks, then the attention with each query tile's online-softmax
 * state initialised from its linear part (tcgen05 MMA).
 */
size_t vattn_hybrid_workspace_bytes(int B, int L, int H, int d, int chunk_tokens);
vattn_status vattn_hybrid_chunk(const void* q, const void* k, const void* v, void* o, float* S,
                                float* z, int B, int L, int H, int d, int chunk_tokens,
                                float scale, void* workspace, size_t workspace_bytes,
                                vattn_stream stream);

/*
 * Hybrid chunk attention, general form: the MobileWan page variant (review
 * of "MobileWan", axiom ledger / App. A.3.1: learnable polynomial feature
 * maps of degree 3 for phi_q and phi_k, softmax chunks overlapping the
 * previous chunk by T_o frames).
 *   fmap VATTN_FMAP_ELU1: phi(x) = elu(x) + 1 (coef unused, may be NULL);
 *   fmap VATTN_FMAP_POLY3: phi_q(x) = a0 + a1 x + a2 x^2 + a3 x^3 with
 *     (a0..a3) = coef[(0 * H + h) * 4 ..], phi_k likewise from
 *     coef[(1 * H + h) * 4 ..]; coef: device fp32 [2][H][4], 16-byte aligned.
 *   overlap_tokens ov >= 0: the softmax part of chunk c covers the keys
 *     [max(0, c * ct - ov), min(L, (c + 1) * ct)) -- its chunk and the last
 *     ov tokens before it -- and the linear part the keys before that window
 *     (plus the incoming state).  The overlap reaches back inside this call
 *     only: chunk 0 has none.  S, z leave as the state after all L tokens.
 *   workspace: vattn_hybrid_workspace_bytes_ex(...) bytes.
 * With fmap ELU1 and ov = 0 this is vattn_hybrid_chunk.
 */
typedef enum { VATTN_FMAP_ELU1 = 0, VATTN_FMAP_POLY3 = 1 } vattn_feature_map;
size_t vattn_hybrid_workspace_bytes_ex(int B, int L, int H, int d, int chunk_tokens, int overlap_tokens);
vattn_status vattn_hybrid_chunk_ex(const void* q, const void* k, const void* v, void* o, float* S, float* z, int B,
                                   int L, int H, int d, int chunk_tokens, int overlap_tokens, float scale,
                                   vattn_feature_map fmap, const float* coef, void* workspace,
                                   size_t workspace_bytes, vattn_stream stream);

/*
 * The state part of vattn_hybrid_chunk as two separate calls, for callers
 * that advance the recurrent state without computing outputs (MobileWan's
 * RNN form of causal linear attention: S_{c+1} = S_c + phi(K_c)^T V_c,
 * z_{c+1} = z_c + sum phi(k)).  Same workspace and layouts as
 * vattn_hybrid_chunk:
 *  - vattn_hybrid_delta writes, for every chunk c of k/v ([B][L][H][d]
 *    bf16), dS_c = phi(K_c)^T V_c (fp32 [C][B][H][d][d]) and
 *    dz_c = sum phi(k) (fp32 [C][B][H][d]) into the workspace (tensor-core
 *    MMA, one pass over K and V);
 *  - vattn_hybrid_scan then replaces them in place by the exclusive prefix
 *    S_c = S_in + sum_{c' < c} dS_c' (same for z) and leaves S, z (in/out)
 *    as the state after the last chunk (one pass of coalesced 16-byte
 *    loads and stores).
 */
vattn_status vattn_hybrid_delta(const void* k, const void* v, int B, int L, int H, int d, int chunk_tokens,
                                void* workspace, size_t workspace_bytes, vattn_stream stream);
vattn_status vattn_hybrid_scan(float* S, float* z, int B, int L, int H, int d, int chunk_tokens, void* workspace,
                               size_t workspace_bytes, vattn_stream stream);

/*
 * vattn_hybrid_chunk without a caller workspace.  The pages have no
 * counterpart: this entry point exists for callers that cannot call
 * cudaMalloc — for instance plug-ins whose host application owns every
 * device allocation, or code that runs where no allocator is reachable —
 * and so cannot supply the scratch that vattn_hybrid_chunk needs.
 *
 * Same arguments and results as vattn_hybrid_chunk, minus the workspace.
 * The scratch (per-chunk state deltas and prefixes) lives instead in one
 * static device array of VATTN_HYBRID_NOALLOC_MAX_BYTES inside libvattn,
 * which every GPU that loads the library holds until the process exits.
 * The call allocates nothing.
 *  - A shape needing more than VATTN_HYBRID_NOALLOC_MAX_BYTES of scratch
 *    (vattn_hybrid_workspace_bytes) is rejected with VATTN_ERR_UNSUPPORTED
 *    before anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - All calls share the one array, which keeps the previous call's
 *    contents; each call writes every scratch element before reading it.
 *    Calls whose kernels overlap on the GPU (e.g. on two streams) race on
 *    the array: order them on one stream or with events.
 */
#define VATTN_HYBRID_NOALLOC_MAX_BYTES ((size_t)32 << 20)
vattn_status vattn_hybrid_chunk_noalloc(const void* q, const void* k, const void* v, void* o, float* S,
                                        float* z, int B, int L, int H, int d, int chunk_tokens,
                                        float scale, vattn_stream stream);

/* Synchronise `stream`, then read and clear the device status word:
   VATTN_ERR_TIMEOUT if a kernel gave up on a wait since the last check. */
vattn_status vattn_check(vattn_stream stream);

const char* vattn_status_string(vattn_status status);
/* Human-readable detail of the last error on the calling thread. */
const char* vattn_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* VATTN_H_ */
