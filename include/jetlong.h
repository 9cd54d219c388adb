/*
 * jetlong.h -- C ABI of libjetlong: Jet-Long dynamic bifocal RoPE causal
 * attention on NVIDIA B200 (sm_100a).
 *
 * Method ("Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
 * RoPE", gist.science/it/paper/2607.07740):
 *   - Metodologia 1 "RoPE Bifocale Dinamico": for a query at position i and a
 *     key at position j, pairs closer than a local window w0 (i - j < w0) use
 *     classic RoPE at the exact positions i and j; all other pairs use RoPE at
 *     the aliased positions f(i), f(j) with f(x) = floor(x / G) and
 *     G = max(1, ceil(L / w_pretrained)) recomputed from the current length L.
 *   - Metodologia 2 "Meccanismi di Efficienza dell'Inferenza": the KV cache
 *     keeps unrotated base keys and is never rewritten; the rotations are
 *     applied on the fly (rotations compose additively); both branches feed one
 *     exact softmax (the pages reach it by an inclusion-exclusion merge of three
 *     attention passes; this library computes the same routed result in one
 *     fused pass with a per-element branch select on boundary tiles).
 *
 * Conventions shared by every entry point
 *   - Tensors are contiguous row-major.  Prefill: q, out [B, Hq, L, d];
 *     k, v [B, Hkv, L, d].  Decode: q, out [B, Hq, d]; kcache, vcache
 *     [B, Hkv, Lcap, d] with rows [0, L) valid.
 *   - q, k and the caches hold UNROTATED ("raw") vectors: the library applies
 *     every rotation.  Frequencies theta_m = rope_theta^(-2m/d), m < d/2,
 *     half-split pairing (x_m, x_{m+d/2}).  Grouped-query attention: q head h
 *     reads kv head h / (Hq / Hkv).  Softmax is softmax(scale * logit), base e.
 *   - Element type: JETLONG_BF16 (q, k, v, caches and out are bf16; tensor-core
 *     path for prefill) or JETLONG_FP32 (all fp32; CUDA-core fp32 path).
 *     Accumulation is fp32 in both.
 *   - Input range (bf16): q and k may hold any finite bf16 values whose logits
 *     scale * <q, k> are finite in fp32.  The rotated Q K^T operands are
 *     rounded to fp16 (11-bit significand) after a power-of-two scaling chosen
 *     from the data: the prefill scales all queries and all keys of a call so
 *     the largest of each lies in [2^13, 2^14) (inputs more than 2^27 below the
 *     largest of their tensor lose relative precision, negligible in any
 *     logit); the decode scales each query head, and each key row of a key
 *     block whose unscaled logits would not be finite.  The scales are exact
 *     and undone in the softmax.  v: |v| below ~1e36 (P.V accumulates in fp32).
 *     NaN inputs give NaN outputs.
 *   - All pointers named d_* or tensor pointers are DEVICE memory owned by the
 *     caller (jetlong_prefill_streamed also takes host buffers, named *_host).
 *     The library never writes q, k, v or the caches (jetlong_prefill_streamed
 *     fills the device staging buffers it is given) and allocates no device
 *     memory in any call.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) on the current device.
 *   - Errors: every entry point returning int returns a jetlong_status.
 *     Arguments are validated on the host before any launch; on failure nothing
 *     is launched and jetlong_last_error() describes the problem.
 */
#ifndef JETLONG_H
#define JETLONG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { JETLONG_BF16 = 0, JETLONG_FP32 = 1 } jetlong_dtype;

typedef enum {
    JETLONG_OK = 0,
    JETLONG_ERR_INVALID_ARG = 1, /* bad pointer, size or parameter          */
    JETLONG_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d)      */
    JETLONG_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed    */
    JETLONG_ERR_TIMEOUT = 4      /* a bounded device wait gave up           */
} jetlong_status;

/* Dynamic group size G = max(1, ceil(L / w_pretrained)) (Metodologia 1,
 * display equation).  Pure host function, int64 arithmetic.  Returns -1 if
 * L < 0 or w_pretrained < 1. */
int64_t jetlong_group_size(int64_t L, int64_t w_pretrained);

/* Aliased position map of Metodologia 1: d_out[x] = floor(x / G) for
 * x in [0, L), G = jetlong_group_size(L, w_pretrained).  d_out: device int32
 * array of L elements.  L must be in [1, 2^31 - 1].  Asynchronous on stream. */
int jetlong_position_map(int32_t* d_out, int64_t L, int64_t w_pretrained, void* stream);

/* Prefill: routed causal attention of every query row of a length-L sequence
 * against keys [0, i] with one G for the call (from this L).
 *   q [B,Hq,L,d], k/v [B,Hkv,L,d] raw inputs; out [B,Hq,L,d] written.
 *   w0 >= 0 local window (w0 = 0: every pair remote; w0 >= L: every pair local);
 *   w_pretrained >= 1; rope_theta > 1; scale > 0 and finite.
 *   d must be 64 or 128 (else JETLONG_ERR_UNSUPPORTED); Hq % Hkv == 0.
 * Sizes: B*Hq*L*d < 2^31 per tensor is NOT required; L < 2^31.
 * bf16 device memory: the call rotates every key once, to its exact and to its
 * aliased position, into fp16 copies (B*Hkv*L*d*2 bytes each; one copy when
 * G = 1) that the attention kernel loads tile by tile.  They live in a
 * stream-ordered pool the library keeps per device: allocated and freed on
 * `stream` around the kernels, reused by later calls, and reserved until the
 * process exits.  The first bf16 prefill call on a device creates the pool:
 * make it before any stream capture (later calls allocate from the pool in
 * stream order, which a capture records).  If the pool cannot grow the call
 * returns JETLONG_ERR_CUDA before any launch of the attention kernel.  The chunked, variable-length,
 * three-pass and streamed calls do the same per launch. */
int jetlong_prefill(const void* q, const void* k, const void* v, void* out,
                    int B, int Hq, int Hkv, int L, int d,
                    int w0, int w_pretrained, double rope_theta, float scale,
                    jetlong_dtype dtype, void* stream);

/* Chunked prefill: the C new query rows of a sequence at positions
 * [P, P + C) attend keys [0, i] of a cache that already holds the previous P
 * keys and the chunk's own C keys, with G from the total length L = P + C
 * (Metodologia 1: G follows the current length; a prompt can be processed in
 * chunks that cross multiples of w_pretrained).  Row i's result equals row i of
 * jetlong_prefill over the whole length-L sequence.
 *   q [B,Hq,C,d] raw queries of the chunk; out [B,Hq,C,d] written.
 *   kcache/vcache [B,Hkv,Lcap,d] raw keys/values, rows [0, P + C) valid (the
 *   caller writes the chunk's keys/values at rows [P, P + C) first); rows
 *   >= P + C are never read into the result.
 *   P >= 0, C >= 1, P + C <= Lcap; other arguments as jetlong_prefill
 *   (jetlong_prefill is this call with P = 0, C = Lcap = L). */
int jetlong_prefill_chunk(const void* q, const void* kcache, const void* vcache, void* out,
                          int B, int Hq, int Hkv, int P, int C, int Lcap, int d,
                          int w0, int w_pretrained, double rope_theta, float scale,
                          jetlong_dtype dtype, void* stream);

/* Variable-length batch: B independent sequences of lengths lens[b] (host
 * array, 1 <= lens[b] <= Lmax), each with its own G = G(lens[b]) (Metodologia
 * 1: G follows each sequence's current length), in padded tensors
 *   q, out [B,Hq,Lmax,d], k, v [B,Hkv,Lmax,d]: rows [0, lens[b]) of sequence b
 *   are used; out rows >= lens[b] are not written.  Padding rows of v must
 *   hold finite values (they meet P = 0 in the P.V product).
 *   lse (optional, may be NULL): float [B,Hq,Lmax] device array, 4-byte
 *   aligned; row i of sequence b receives log sum_j exp(scale * logit_ij)
 *   (natural log; the statistic an LSE merge of partial attentions needs).
 * Other arguments and errors as jetlong_prefill.  bf16: one prefill launch
 * (after a range scan and a key rotation) per 64 sequences, its grid over the
 * query blocks of all of them, heaviest first; padding rows of q and k may
 * hold anything.  fp32: one launch per sequence. */
int jetlong_prefill_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                           int B, int Hq, int Hkv, const int32_t* lens, int Lmax, int d,
                           int w0, int w_pretrained, double rope_theta, float scale,
                           jetlong_dtype dtype, void* stream);

/* The pages' own formulation of the prefill (Metodologia 2, inclusion-
 * exclusion): three standard attention passes -- A: window pairs (i - j < w0)
 * at the exact positions, B: all causal pairs at the aliased positions, C:
 * window pairs at the aliased positions -- merged per row with their softmax
 * denominators, out = (e^lA O_A + e^lB O_B - e^lC O_C) / (e^lA + e^lB - e^lC).
 * The result equals jetlong_prefill's up to rounding; it exists to compare
 * the two forms.  Arguments as jetlong_prefill, plus a device workspace of at
 * least jetlong_prefill_ie_workspace_size(B, Hq, L, d, dtype) bytes (16-byte
 * aligned, caller-owned; the three pass outputs in fp32 -- the merge subtracts
 * nearly equal terms, so they are not rounded to bf16 first -- and their
 * LSEs).  Three passes (each a range scan and a prefill launch for bf16) and
 * the merge; when w0 = 0, pass B alone, written into out. */
size_t jetlong_prefill_ie_workspace_size(int B, int Hq, int L, int d, jetlong_dtype dtype);
int jetlong_prefill_ie(const void* q, const void* k, const void* v, void* out,
                       int B, int Hq, int Hkv, int L, int d,
                       int w0, int w_pretrained, double rope_theta, float scale,
                       jetlong_dtype dtype, void* workspace, size_t workspace_bytes, void* stream);

/* Prefill from host buffers with the transfers overlapped: the sequence is
 * processed as min(nchunks, ceil(L / 128)) chunks of query rows (whole 128-row
 * blocks; the first and the last chunk a quarter of the size of the others,
 * since nothing overlaps their copy in and out), and while
 * chunk c computes (jetlong_prefill_chunk semantics over the rows uploaded so
 * far) the rows of chunk c + 1 travel host -> device and those of chunk c - 1
 * device -> host, on two copy streams the library keeps per device.
 *   q_host, k_host, v_host, out_host: host tensors [B,H,L,d] (page-locked
 *   memory for the copies to overlap); q_dev, k_dev, v_dev, out_dev: device
 *   tensors of the same shapes, owned by the caller, 16-byte aligned.
 *   nchunks >= 1; other arguments as jetlong_prefill.
 * Asynchronous: work queued on `stream` afterwards runs after out_host is
 * complete.  Same result as copying in, jetlong_prefill, copying out.  If the
 * call fails part-way, work queued on `stream` afterwards still runs only
 * after every copy the call did queue (so the buffers can be freed or reused
 * in stream order). */
int jetlong_prefill_streamed(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                             void* q_dev, void* k_dev, void* v_dev, void* out_dev,
                             int B, int Hq, int Hkv, int L, int d,
                             int w0, int w_pretrained, double rope_theta, float scale,
                             jetlong_dtype dtype, int nchunks, void* stream);

/* Bytes of device workspace jetlong_decode needs for any L <= Lcap with these
 * sizes (partial softmax states of the key splits plus merge counters).
 * Returns 0 for invalid sizes. */
size_t jetlong_decode_workspace_size(int B, int Hq, int Hkv, int Lcap, int d);

/* Decode: one new query per (b, h) at position i = L - 1 attending cache rows
 * [0, L), with G recomputed from this L (so G changes as generation crosses a
 * multiple of w_pretrained while the cache is untouched, Metodologia 2).  The
 * caller appends the new token's raw key/value at row L - 1 beforehand.
 *   q [B,Hq,d] raw, kcache/vcache [B,Hkv,Lcap,d] raw, out [B,Hq,d] written.
 *   1 <= L <= Lcap.  workspace: device memory of at least
 *   jetlong_decode_workspace_size(B,Hq,Hkv,Lcap,d) bytes, 16-byte aligned,
 *   owned by the caller; its contents on entry do not matter.  Two calls that
 *   share one workspace must not overlap on the device. */
int jetlong_decode(const void* q, const void* kcache, const void* vcache, void* out,
                   int B, int Hq, int Hkv, int L, int Lcap, int d,
                   int w0, int w_pretrained, double rope_theta, float scale,
                   jetlong_dtype dtype, void* workspace, size_t workspace_bytes,
                   void* stream);

/* Decode over a standard RoPE key cache (the pages' own decode mechanism,
 * Metodologia 2: the cache keeps every key at its base rotation and the
 * bifocal positions are reached by correcting rotations, since rotations
 * compose additively).  Row j of kcache holds the key already rotated to its
 * exact position j, as an ordinary RoPE model writes it; vcache is unchanged.
 * A local key (i - j < w0) is used as stored, a remote key is rotated by
 * f(j) - j (<= 0) to reach f(j); the query is rotated to i or f(i) as in
 * jetlong_decode.  Same arguments, sizes, workspace, ownership and errors as
 * jetlong_decode; the result equals jetlong_decode on the raw keys up to the
 * rounding of the stored rotated keys. */
int jetlong_decode_rope_cache(const void* q, const void* kcache, const void* vcache, void* out,
                              int B, int Hq, int Hkv, int L, int Lcap, int d,
                              int w0, int w_pretrained, double rope_theta, float scale,
                              jetlong_dtype dtype, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Allocation-free decode.  The paper has no counterpart to this entry point:
 * it exists for callers that cannot allocate device memory at all (a serving
 * runtime whose caching allocator must not grow, code running in a host
 * callback, or a host framework that hands this library only the step's
 * tensors), so they cannot supply jetlong_decode's workspace.
 *
 * Same arguments, semantics and results as jetlong_decode without the
 * workspace: the split partials and merge counters live in one fixed device
 * array of JETLONG_DECODE_NOALLOC_SCRATCH_BYTES inside the library, which every
 * GPU that loads the library holds until the process exits.  The call allocates
 * nothing (no cudaMalloc, no allocating library routine).
 *   - The first call on each device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - Problems whose scratch exceeds the array are rejected with
 *     JETLONG_ERR_INVALID_ARG before any launch (the message gives the bytes
 *     needed); use jetlong_decode with a workspace for them.
 *   - All calls on a device share the array and leave their contents in it.
 *     Calls that overlap on the GPU (e.g. on two streams without ordering
 *     between them) race on the array and give wrong results: serialise them. */
#define JETLONG_DECODE_NOALLOC_SCRATCH_BYTES (4u << 20)
int jetlong_decode_noalloc(const void* q, const void* kcache, const void* vcache, void* out,
                           int B, int Hq, int Hkv, int L, int Lcap, int d,
                           int w0, int w_pretrained, double rope_theta, float scale,
                           jetlong_dtype dtype, void* stream);

/* Synchronises `stream`, then reads and clears the library's device error
 * word, set by a kernel whose bounded wait expired (the kernel then returned
 * without finishing its tile).  Returns JETLONG_OK, JETLONG_ERR_TIMEOUT or
 * JETLONG_ERR_CUDA. */
int jetlong_device_status(void* stream);

/* Self test of the failure-detection path (the pages have no counterpart):
 * launches one small kernel that waits on a barrier nothing arrives at, using
 * the same bounded-wait helper as the attention kernels with a ~1 ms limit.
 * The wait expires, the kernel sets the device error word and returns, so the
 * next jetlong_device_status(stream) reports JETLONG_ERR_TIMEOUT (and clears
 * the word).  No fault, no hang; the context stays usable.  Returns
 * JETLONG_OK or JETLONG_ERR_CUDA (launch failure). */
int jetlong_selftest_wait_timeout(void* stream);

/* Failure-detection test hook (the pages have no counterpart).  Arms a
 * one-shot fault injection for the next attention call made on this host
 * thread: the kernel it launches withholds one barrier arrival, chosen by
 * `site`, and every bounded wait of that launch gives up after `wait_cycles`
 * SM cycles instead of the normal ~0.5 s (prefill) / ~2 s (decode).  The
 * waits that depend on the withheld arrival expire; the kernel records a code
 * in the device error word, its roles stop, drain their own copies and MMAs,
 * release tensor memory and return, so the next jetlong_device_status reports
 * JETLONG_ERR_TIMEOUT and the context stays usable.  The output of the
 * sabotaged call is undefined.  No fault, trap or unbounded wait is involved.
 *   JETLONG_INJECT_PREFILL_KEY_TILE: bf16 prefill (both tensor-core kernels):
 *       the first key tile of every work unit is never released to the MMA
 *       issuer.
 *   JETLONG_INJECT_DECODE_COPY: bf16 decode: the first K/V stage of every
 *       key split is never loaded.
 * The hook is consumed by the next prefill or decode call of this thread that
 * passes argument validation (whatever its dtype; the fp32 kernels ignore it);
 * JETLONG_INJECT_NONE disarms it.  wait_cycles in [1e4, 4e9] (ignored for
 * JETLONG_INJECT_NONE).  Returns JETLONG_OK or JETLONG_ERR_INVALID_ARG. */
#define JETLONG_INJECT_NONE 0
#define JETLONG_INJECT_PREFILL_KEY_TILE 1
#define JETLONG_INJECT_DECODE_COPY 2
int jetlong_debug_inject_timeout(int site, long long wait_cycles);

/* Test hooks (the pages have no counterpart): the device helpers of the
 * attention kernels on their own, for checks against host computations.
 *
 * jetlong_debug_rope_phase: d_out[2 (i d/2 + m) + {0, 1}] = (cos, sin) of
 * d_pos[i] * theta_m, theta_m = rope_theta^(-2m/d), m < d/2, as the kernels
 * form it (exact fixed-point turn fraction, then sincospif when `accurate`,
 * else __sincosf).  d_pos: n uint32 positions; d_out: 2 n d/2 floats (device).
 *
 * jetlong_debug_tile_plan: for the query blocks qb (128 rows each) of rows
 * [P, P + C) against keys [0, L = P + C) with window w0: d_plan[3 qb + {0,1,2}]
 * = (nR, kE0, nkb) -- the remote-phase tiles are key blocks [0, nR), the
 * exact-phase tiles [kE0, nkb) -- and d_cls[qb max_kb + kb] (kb < min(nkb,
 * max_kb)) the class of tile (qb, kb): 0 every causal pair remote, 1 every pair
 * local, 2 both.  Device arrays of 3 ceil(C / 128) int32 and ceil(C / 128)
 * max_kb int8.
 *
 * jetlong_debug_ex2: d_out[i] = 2^d_y[i] as the one-CTA prefill's softmax
 * forms part of its exponentials on the FMA pipe (round to an integer n,
 * cubic in the remainder, exponent bits for 2^n; inputs below -127 give 0,
 * NaN stays NaN).  Meant for y <= 2^7, the softmax's range.  d_y, d_out:
 * device float arrays of n elements, n even.
 *
 * jetlong_debug_rope_keys: the bf16 prefill's key rotation pass on its own --
 * the range scan of d_k, then d_kl[z][j] = R(j) k[z][j] 2^e and (unless d_kr
 * is NULL) d_kr[z][j] = R(floor(j / G)) k[z][j] 2^e, as fp16, with 2^e the
 * power-of-two key scale the prefill would use (e = 13 - floor(log2 max|k|),
 * clamped to [-100, 100]; 0 for an all-zero or non-finite k).  d_k: bf16
 * [planes][L][d]; d_kl, d_kr: fp16 of the same shape, 16-byte aligned; *h_exp
 * (host) receives e, so this call synchronises the stream.
 *
 * All return JETLONG_OK, JETLONG_ERR_INVALID_ARG or JETLONG_ERR_CUDA;
 * asynchronous on stream unless stated. */
int jetlong_debug_rope_phase(const uint32_t* d_pos, int64_t n, int d, double rope_theta, int accurate,
                             float* d_out, void* stream);
int jetlong_debug_tile_plan(int P, int C, int w0, int max_kb, int32_t* d_plan, int8_t* d_cls, void* stream);
int jetlong_debug_ex2(const float* d_y, int64_t n, float* d_out, void* stream);
int jetlong_debug_rope_keys(const void* d_k, int planes, int L, int d, int G, double rope_theta, void* d_kl,
                            void* d_kr, int* h_exp, void* stream);

/* Message for the last failing call on this host thread ("" if none). */
const char* jetlong_last_error(void);

/* Number of kernels this library has launched in this process. */
uint64_t jetlong_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* JETLONG_H */
