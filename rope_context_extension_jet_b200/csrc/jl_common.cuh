// jl_common.cuh -- declarations shared by the libjetlong translation units.
//
// RoPE phase arithmetic.  The rotation angle of pair m at position p is
// p * theta_m with theta_m = rope_theta^(-2m/d) (standard RoPE frequencies,
// half-split pairing; the pages evaluate Qwen3 models, which use this form).
// Positions reach 131071 and theta_0 = 1 rad/token, so the plain fp32 product
// p * theta_m would be off by ~1e-2 rad.  Instead the host stores
// omega_m = theta_m / (2 pi) as an unsigned 0.64 fixed-point fraction of a
// turn; the device forms the angle's fractional turn exactly as the low 64 bits
// of p * omega_m (only the top 32 are needed), converts that to an fp32 value
// in [-0.5, 0.5) and calls CUDA's sincospif / __sincosf on it.  The resulting
// angle error is ~1e-7 rad at any position (rounding of the fp32 turn value).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "jetlong.h"

namespace jl {

constexpr int kMaxHalf = 64;  // d <= 128

// omega_m = theta_m / (2 pi) in 0.64 fixed point, split into 32-bit words.
struct RopeTurns {
    uint32_t hi[kMaxHalf];
    uint32_t lo[kMaxHalf];
};

void make_rope_turns(RopeTurns* t, int d, double rope_theta);

// Fractional turn of p * omega (exact modulo 2^-32 turn), as fp32 in [-0.5, 0.5).
__device__ __forceinline__ float rope_turn(uint32_t p, uint32_t w_hi, uint32_t w_lo)
{
    uint32_t top = p * w_hi + __umulhi(p, w_lo);
    return (float)(int32_t)top * 2.3283064365386963e-10f;  // 2^-32
}

// Accurate cos/sin of the angle of pair m at position p (sincospif, ~1 ulp).
__device__ __forceinline__ void rope_cs_accurate(uint32_t p, uint32_t w_hi, uint32_t w_lo,
                                                 float& c, float& s)
{
    float t = rope_turn(p, w_hi, w_lo);
    sincospif(2.0f * t, &s, &c);
}

// Fast cos/sin (hardware approximations on the reduced angle in [-pi, pi);
// absolute error ~5e-7).
__device__ __forceinline__ void rope_cs_fast(uint32_t p, uint32_t w_hi, uint32_t w_lo,
                                             float& c, float& s)
{
    float t = rope_turn(p, w_hi, w_lo);
    __sincosf(6.28318530717958647692f * t, &s, &c);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    __half2 r = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}

template <typename T> __device__ __forceinline__ float load_elem(const T* p);
template <> __device__ __forceinline__ float load_elem<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p)
{
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void store_elem(T* p, float x);
template <> __device__ __forceinline__ void store_elem<float>(float* p, float x) { *p = x; }
template <> __device__ __forceinline__ void store_elem<__nv_bfloat16>(__nv_bfloat16* p, float x)
{
    *p = __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// Host-side launch plumbing shared by the translation units.

// Prefill of query rows at positions [P, P + C) against keys [0, L), L = P + C
// (a whole sequence: P = 0, C = L).  q and out hold Cst >= C rows per (b, head)
// (rows [0, C) used); k and v hold Lcap >= L rows per (b, kv head), rows [0, L)
// valid.  lse (optional, may be null): Cst floats per (b, head), row r receives
// the natural log of row r's softmax denominator.
struct PrefillProblem {
    const void *q, *k, *v;
    void* out;
    float* lse;
    int B, Hq, Hkv, L, d, w0;
    int P, C, Cst, Lcap;
    // -1: the routed (bifocal) attention.  0 / 1: a plain windowed attention
    // over the pairs with i - j < w0 only, every pair rotated to its exact (0)
    // or aliased (1) positions (passes of the pages' inclusion-exclusion form).
    int window_rot;
    int G;             // dynamic group size for this call (fits int: G <= L)
    float scale_log2;  // scale * log2(e): logits kept in base-2 units
    RopeTurns turns;
    int* dev_error;    // device error word (bounded waits)
    long long wait_cycles;  // limit of every bounded wait of the attention roles
    int inject;             // failure-detection test hook (kInjectNone in normal calls)
    // bf16: two words (largest |q|, largest |k| as bf16 magnitude bits) written
    // by launch_range_scan on the same stream before the prefill kernel
    const uint32_t* range;
    // bf16 variable-length batch in one launch (vl_n > 0, at most 64
    // sequences): lengths and group sizes of sequences 0..vl_n-1; B = vl_n, P = 0,
    // q / out / k / v planes of Cst = Lcap = L = the longest length (L, C are
    // then the batch maximum)
    int vl_n;
    int vl_len[64], vl_G[64];
    // bf16: write out as fp32 rows (the three-pass form's intermediate passes)
    int out_f32;
    // bf16: the call's keys rotated once by launch_rope_keys, fp16 planes of L
    // rows: to their exact positions (krot_l) and to floor(j / G) (krot_r,
    // equal to krot_l when G = 1 throughout)
    const void* krot_l;
    const void* krot_r;
};

struct DecodeProblem {
    const void *q, *kc, *vc;
    void* out;
    int B, Hq, Hkv, L, Lcap, d, w0;
    int G;
    int rope_cache;  // 0: raw key rows; 1: key row j stored rotated to its exact position j
    float scale_log2;
    RopeTurns turns;
    void* workspace;
    size_t workspace_bytes;
    int* dev_error;
    long long wait_cycles;
    int inject;
};

// Failure-detection test hook: the barrier arrival a launch withholds (the
// values of jetlong_debug_inject_timeout's `site`).
enum {
    kInjectNone = 0,
    kInjectPrefillKeyTile = JETLONG_INJECT_PREFILL_KEY_TILE,  // bf16 prefill: the first key tile is never released
    kInjectDecodeCopy = JETLONG_INJECT_DECODE_COPY,           // bf16 decode: the first K/V stage is never loaded
};
// Normal limits: ~0.5 s for the prefill roles, ~2 s for the decode (every wait
// is on work of the same CTA or CTA pair).
constexpr long long kPrefillWaitCycles = 1000000000ll;
constexpr long long kDecodeWaitCycles = 4000000000ll;

// Returns cudaSuccess or the launch error; each adds its launches to *nlaunch.
cudaError_t launch_prefill_simt(const PrefillProblem& p, jetlong_dtype dt, cudaStream_t s,
                                int* nlaunch);
cudaError_t launch_prefill_tc(const PrefillProblem& p, cudaStream_t s, int* nlaunch);
cudaError_t launch_decode(const DecodeProblem& p, jetlong_dtype dt, cudaStream_t s, int* nlaunch);
// Same decode with its scratch in the library's fixed device array; *need_bytes
// receives the scratch this problem needs (cudaErrorInvalidValue if too large).
cudaError_t launch_decode_noalloc(const DecodeProblem& p, jetlong_dtype dt, cudaStream_t s,
                                  int* nlaunch, size_t* need_bytes);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Lcap, int d);
cudaError_t launch_position_map(int32_t* out, int L, int G, cudaStream_t s, int* nlaunch);
// Inclusion-exclusion merge of three attention passes (A, B, C) with their
// per-row LSEs: out = (e^lA O_A + e^lB O_B - e^lC O_C) / (e^lA + e^lB - e^lC).
// The pass outputs are fp32 rows; out has the element type dt.
cudaError_t launch_ie_merge(const void* oa, const void* ob, const void* oc, const float* la, const float* lb,
                            const float* lc, void* out, long long rows, int d, jetlong_dtype dt,
                            cudaStream_t s, int* nlaunch);
cudaError_t launch_wait_selftest(int* dev_error, long long limit_cycles, cudaStream_t s, int* nlaunch);
// Largest magnitude of the used rows of q (planes of Cst rows, rows [0, C)) and
// of k (planes of Lcap rows, rows [0, L)), bf16, as 15-bit magnitude bits into
// range[0] and range[1] (zeroed first on the stream).
// Test hooks (debug_kernels.cu): the phase helpers and the tile plan on their own.
cudaError_t launch_rope_phase(const uint32_t* pos, long long n, int d, const RopeTurns& turns, int accurate,
                              float* out, cudaStream_t s, int* nlaunch);
cudaError_t launch_ex2_poly(const float* y, long long n, float* out, cudaStream_t s, int* nlaunch);
cudaError_t launch_tile_plan(int P, int C, int L, int w0, int max_kb, int32_t* plan, int8_t* cls, cudaStream_t s,
                             int* nlaunch);
// rows (optional): per-sequence row counts of a variable-length batch, plane pl
// of q (k) belonging to sequence pl / hq (pl / hkv).
struct ScanRows {
    int n, hq, hkv;
    int len[64];
};
cudaError_t launch_range_scan(const void* q, int C, int Cst, int q_planes, const void* k, int L, int Lcap,
                              int k_planes, int d, uint32_t* range, cudaStream_t s, int* nlaunch,
                              const ScanRows* rows = nullptr);

// Keys of a bf16 prefill call rotated once to their exact and aliased
// positions (rope_keys.cu): bytes of one fp16 copy, whether the aliased copy
// differs from the exact one (some G > 1), and the launch that writes kl (and
// kr unless null) after the call's range scan on the same stream.
size_t rope_keys_bytes(const PrefillProblem& p);
bool rope_keys_need_remote(const PrefillProblem& p);
cudaError_t launch_rope_keys(const PrefillProblem& p, void* kl, void* kr, cudaStream_t s, int* nlaunch);

}  // namespace jl
