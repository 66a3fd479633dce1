/*
 * sdpa.h -- C ABI of the B200 (sm_100a) fused scaled-dot-product attention
 * library: forward and backward of
 *
 *     O = softmax(scale * Q K^T + bias, masked) V
 *
 * Definition: codelab "jax-gpu-05-attention-gpu", section 1 (how attention
 * works: score, scale + softmax, weighted sum, output shaped like Q) and
 * section 4 (the naive reference); Medium "Simplified Explanation of
 * Attention ...", Steps 1-4 of "Scaled Dot Product Operation".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  Q, K, V, O, dO, dQ, dK, dV are bf16 tensors in (batch, sequence,
 *   head, head_dim) order -- the (B, T, N, H) layout of the codelab, section
 *   3 -- given by element strides; head_dim is contiguous.  Q, O, dO and dQ
 *   share the strides sq_*, K, V, dK and dV share skv_*.  Queries have L rows,
 *   keys and values Lk (Lk = L for self-attention; cross-attention, as in a
 *   T5 decoder attending to its encoder, may differ).  Positions of both
 *   sequences count from 0: the causal and window masks and the relative-
 *   position biases compare the query index i with the key index j as they
 *   are.  LSE is float32 [B, Hq, L], contiguous.  Packed variable-length
 *   batches (sdpa_fwd_varlen / sdpa_bwd_varlen) lay the sequences end to end
 *   along one sequence axis instead, described by sdpa_varlen.
 * Heads.  Hq query heads share Hkv key/value heads in contiguous groups:
 *   query head h reads KV head h / (Hq / Hkv) (MHA Hkv = Hq, GQA, MQA
 *   Hkv = 1; codelab section 9).  Hq % Hkv must be 0.
 * Supported.  head_dim d in {64, 128}; 1 <= L, Lk < 2^30; B, Hq <= 65535;
 *   ceil(L / 128) * Hq * B < 2^31 (query tiles are counted in 32 bits);
 *   every bf16 base pointer 16-byte aligned; every stride a multiple of 8
 *   elements (16 bytes) except the contiguous head_dim.  Anything else returns SDPA_ERR_UNSUPPORTED or
 *   SDPA_ERR_INVALID_ARG before any work is queued.
 * Ownership.  The caller owns every buffer.  No entry point allocates,
 *   frees, or synchronises the stream, except sdpa_read_device_status.
 *   Outputs (O, LSE, dQ, dK, dV) are fully overwritten; no pre-zeroing.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream); work is queued on it and the call returns without waiting.
 *   Device pointers must belong to the current CUDA device.
 * Errors.  Argument errors are reported synchronously before any launch;
 *   launch failures return SDPA_ERR_CUDA.  Waits inside the kernels are
 *   bounded: a wait that runs out records SDPA_ERR_TIMEOUT in a per-device
 *   status word (read with sdpa_read_device_status) and the kernel returns
 *   instead of hanging.
 * Accuracy.  bf16 inputs and outputs with float32 accumulation.  Against an
 *   exact (float64) evaluation, O, dQ, dK and dV are within
 *   1e-2 + 1e-2 |ref| element-wise and LSE within 1e-3 for N(0, 1) inputs at
 *   scales up to 1 / sqrt(d) (and at smaller or negative scales).  Larger
 *   scales -- T5's historical scale 1, say -- make the softmax peaked, and
 *   the bf16 rounding of dS (the operand of the dQ and dK products) and of
 *   the stored O (in D = rowsum(dO * O)) can then exceed that bound on a few
 *   gradient entries where large terms cancel.
 * Determinism.  Results are bit-identical run to run for identical inputs
 *   and launch configuration: every reduction is in a fixed order and no
 *   floating-point atomics are used (HF transformers issue #31787,
 *   "Transformer models are not deterministic when using Flash Attention 2",
 *   is the problem this guards against).
 */
#ifndef SDPA_B200_SDPA_H
#define SDPA_B200_SDPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sdpa_status_t {
  SDPA_OK = 0,
  SDPA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, stride or alignment  */
  SDPA_ERR_UNSUPPORTED = 2,  /* valid but not built: e.g. head_dim 96        */
  SDPA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small   */
  SDPA_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed           */
  SDPA_ERR_TIMEOUT = 5       /* a bounded in-kernel wait ran out              */
} sdpa_status_t;

/*
 * Mask specification -- replaces a dense mask tensor.  Key j is visible from
 * query i iff
 *     (!causal || j <= i) && (window_left < 0 || j >= i - window_left)
 *                         && (window_right < 0 || j <= i + window_right).
 * Causal masking: codelab section 7.  Causal sliding window (Mistral,
 * window 4096): HF transformers issue #30461, "Slowdown in Training Speed Due
 * to SDPA Mask Fix in Version 4.40.0", whose whole point is that handing this
 * mask over as a dense tensor forfeits skipping fully masked key tiles.  The
 * pages do not say whether the window bound is inclusive; here both bounds
 * are inclusive and a negative bound means unbounded.
 */
typedef struct sdpa_mask_spec {
  int32_t causal;
  int64_t window_left;
  int64_t window_right;
} sdpa_mask_spec;

typedef enum sdpa_bias_kind {
  SDPA_BIAS_NONE = 0,
  SDPA_BIAS_DENSE = 1, /* additive float32 bias[b, h, i, j]                  */
  SDPA_BIAS_T5 = 2,    /* additive table[bucket(j - i), h], bucketed in-kernel */
  SDPA_BIAS_ALIBI = 3, /* additive -slope[h] |j - i|, computed in-kernel       */
  SDPA_BIAS_REL = 4    /* additive table[j - i + Lq - 1, h] (any function of j - i) */
} sdpa_bias_kind;

/*
 * Additive attention bias (catie-aq/flashT5 README: "Full attention biases"
 * and "T5-like relative position encoding biases"; the 3 October 2024
 * "fa2-rpe" item -- linear memory for the T5 bias).  The bias is added after
 * the scale and is not itself scaled; it takes part in LSE.
 *   DENSE: ptr -> float32 with element strides stride_b, stride_h, stride_i
 *          (j contiguous; 0 broadcasts over that index); ptr 16-byte aligned,
 *          stride_b, stride_h, stride_i multiples of 4 (rows are read in
 *          16-byte pieces); stride_i = 0 (one row for every query) ->
 *          SDPA_ERR_UNSUPPORTED.  A value of -inf masks (i, j); a row
 *          with no visible key yields O = 0, LSE = -inf, zero gradients.
 *   T5:    ptr -> float32 table[num_buckets][Hq] (row-major), bucket of the
 *          signed distance j - i by the T5 closed form (Raffel et al. 2020):
 *          bidirectional splits the buckets by sign; 2 <= num_buckets <= 128,
 *          num_buckets even when bidirectional, max_distance > max_exact
 *          (num_buckets/4 when bidirectional, num_buckets/2 otherwise).
 *          Nothing L x L is materialised.
 *   ALIBI: ptr -> float32 slopes[Hq]; bias[h, i, j] = -slopes[h] |j - i|.
 *          The README names ALiBi among its positional schemes without a
 *          formula; this is the linear bias of Press et al. 2022 ("Train
 *          Short, Test Long"), equal to their -m (i - j) on the keys a causal
 *          mask leaves.  Strides and T5 fields are ignored.
 *   REL:   ptr -> float32 table[Lq + Lk - 1][Hq] (row-major); bias[h, i, j]
 *          = table[j - i + Lq - 1][h]: any per-head function of the
 *          distance, looked up per tile like T5 (the general form of T5 and
 *          ALiBi; FIRE enters this way through sdpa_fire_table).  Packed
 *          batches index it with the longest lengths (max_seqlen_q - 1
 *          offset, positions from 0 in each sequence).  Strides and T5
 *          fields are ignored.
 */
typedef struct sdpa_bias_desc {
  int32_t kind; /* sdpa_bias_kind */
  const float* ptr;
  int64_t stride_b, stride_h, stride_i;
  int32_t num_buckets, max_distance, bidirectional;
} sdpa_bias_desc;

typedef struct sdpa_shape {
  int64_t B, L, Hq, Hkv, d;
  int64_t sq_b, sq_l, sq_h;    /* element strides of Q, O, dO, dQ */
  int64_t skv_b, skv_l, skv_h; /* element strides of K, V, dK, dV */
  int64_t Lk;                  /* key / value length; 0 = L */
} sdpa_shape;

/*
 * Packed variable-length sequences (HF transformers issue #30461: the Mistral
 * fine-tune packs its examples, `packing=True`; catie-aq/flashT5 README:
 * dynamic batching to cut padding).  Batch entry b owns query rows
 * [cu_seqlens_q[b], cu_seqlens_q[b + 1]) and key rows [cu_seqlens_k[b],
 * cu_seqlens_k[b + 1]) of one shared sequence axis; its positions count from
 * 0 at its first row and no query attends to another entry's keys.
 *   cu_seqlens_q, cu_seqlens_k: device int32 [B + 1], non-decreasing, first
 *     entry 0, last entry total_q / total_k, read by the kernels (entries
 *     that leave [0, total] or give a sequence longer than max_seqlen make
 *     that entry empty and are reported by sdpa_read_device_status as
 *     SDPA_ERR_UNSUPPORTED).
 *   max_seqlen_q / max_seqlen_k: upper bounds of the lengths (>= 1).
 *   total_q / total_k: rows of the packed axes (>= 1, < 2^30).
 * With a packed batch the shape's B is the number of sequences, its L and Lk
 * and batch strides sq_b / skv_b are ignored: Q, O, dO, dQ are
 * [total_q, Hq, d] with strides sq_l, sq_h, K, V, dK, dV [total_k, Hkv, d]
 * with skv_l, skv_h, and LSE is float32 [Hq, total_q].  Dense biases have no
 * packed form (SDPA_ERR_UNSUPPORTED); T5 and ALiBi biases are relative
 * positions within each sequence.
 */
typedef struct sdpa_varlen {
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  int64_t max_seqlen_q, max_seqlen_k;
  int64_t total_q, total_k;
} sdpa_varlen;

/*
 * Forward.  Writes O (bf16, Q's layout) and LSE[b, h, i] = natural-log
 * log-sum-exp of score row i (float32, -inf for a row with no visible key).
 * bias may be NULL (= no bias); mask may not be NULL.  Fully masked key
 * tiles are never loaded.
 */
sdpa_status_t sdpa_fwd(const sdpa_shape* shape, const void* q, const void* k,
                       const void* v, const sdpa_bias_desc* bias,
                       const sdpa_mask_spec* mask, float scale, void* o,
                       float* lse, void* stream);

/* Forward of a packed variable-length batch (see sdpa_varlen). */
sdpa_status_t sdpa_fwd_varlen(const sdpa_shape* shape, const sdpa_varlen* varlen,
                              const void* q, const void* k, const void* v,
                              const sdpa_bias_desc* bias, const sdpa_mask_spec* mask,
                              float scale, void* o, float* lse, void* stream);

/*
 * Bytes of device workspace sdpa_bwd needs for this shape: the per-row
 * D_i = sum_c dO[i,c] O[i,c] vector (float32, one per LSE entry), rounded
 * up to 256 bytes.  Returns 0 for an invalid shape.
 */
size_t sdpa_bwd_workspace_size(const sdpa_shape* shape, int32_t deterministic);
size_t sdpa_bwd_varlen_workspace_size(const sdpa_shape* shape, const sdpa_varlen* varlen);

/*
 * Backward.  Given Q, K, V, the forward output O and its LSE, and the
 * output gradient dO (Q's layout), writes dQ (Q's layout), dK and dV (K's
 * layout, summed over the query heads that share each KV head).  The pages
 * print no gradient formulas; these are the chain rule of the forward:
 *   P = exp(S - LSE), dP = dO V^T, D_i = rowsum(dO * O), dS = P (dP - D),
 *   dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
 * Three launches: D into the workspace; dQ, one CTA per 128 query rows
 * summing over the key tiles of the mask band in ascending order on chip;
 * dK and dV, one CTA per 128 keys summing over the query tiles and the
 * query heads of its group in a fixed order on chip.  Every sum has a fixed
 * order and none uses floating-point atomics, so repeated calls give
 * bit-identical results (HF transformers issue #31787 is the
 * non-determinism this avoids).
 * deterministic: must be 1 (the only mode built; 0 returns UNSUPPORTED).
 * workspace: device memory of at least sdpa_bwd_workspace_size() bytes,
 * 256-byte aligned, owned by the caller, contents ignored on entry.
 */
sdpa_status_t sdpa_bwd(const sdpa_shape* shape, const void* q, const void* k,
                       const void* v, const void* o, const void* dout,
                       const float* lse, const sdpa_bias_desc* bias,
                       const sdpa_mask_spec* mask, float scale, void* dq,
                       void* dk, void* dv, int32_t deterministic,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * The backward as its three launches, selected by a bitmask: PREPROCESS
 * writes D = rowsum(dO * O) into the workspace; DQ writes dQ and DKDV
 * writes dK and dV, both reading D, so they need a PREPROCESS on the same
 * workspace (with the same O and dO) earlier in stream order; D stays valid
 * for any number of DQ / DKDV launches after it.  sdpa_bwd is
 * sdpa_bwd_phases(SDPA_BWD_ALL, ...).  Arguments as sdpa_bwd; phases == 0
 * or unknown bits -> SDPA_ERR_INVALID_ARG.
 */
#define SDPA_BWD_PREPROCESS 1u
#define SDPA_BWD_DQ 2u
#define SDPA_BWD_DKDV 4u
#define SDPA_BWD_ALL 7u
sdpa_status_t sdpa_bwd_phases(uint32_t phases, const sdpa_shape* shape, const void* q,
                              const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, const sdpa_bias_desc* bias,
                              const sdpa_mask_spec* mask, float scale, void* dq, void* dk,
                              void* dv, int32_t deterministic, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Backward of a packed variable-length batch (see sdpa_varlen); workspace of
 * at least sdpa_bwd_varlen_workspace_size() bytes. */
sdpa_status_t sdpa_bwd_varlen(const sdpa_shape* shape, const sdpa_varlen* varlen,
                              const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, const sdpa_bias_desc* bias,
                              const sdpa_mask_spec* mask, float scale, void* dq, void* dk,
                              void* dv, int32_t deterministic, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Backward without a caller-supplied workspace.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot
 * allocate device memory around the call: kernel hosts and plugin
 * interfaces that hand a library only its input and output buffers and own
 * every other byte of device memory through their own pool, processes held
 * to a hard memory cap where a late allocation can fail mid-step, and
 * latency-bound loops that avoid cudaMalloc / cudaFree because those calls
 * can synchronise the device and stall other streams.
 *
 * Same arguments and results as sdpa_bwd minus the workspace: the workspace
 * lives in a fixed array of SDPA_NOALLOC_SCRATCH_BYTES (16 MiB) compiled into
 * the library, held by every GPU that loads it until the process exits.
 *  - sdpa_bwd_workspace_size(shape) must be <= SDPA_NOALLOC_SCRATCH_BYTES
 *    (4 bytes per LSE entry: B * Hq * L up to 4194304, or Hq times the
 *    packed rows), else SDPA_ERR_WORKSPACE (nothing is launched).
 *  - The first call on a device looks up the array's device address with
 *    that device current (once per device); make that first call before
 *    any stream capture on the device.  A failed lookup -> SDPA_ERR_CUDA.
 *  - Every call, on every stream of a device, shares the one array, which
 *    keeps the contents of the last call (each call writes every entry it
 *    reads before reading it).  Calls whose executions
 *    overlap on the GPU race on it; order them on one stream or with events.
 *  - The looked-up address is cached per device for the life of the
 *    process; it does not survive cudaDeviceReset (or any other teardown of
 *    the device's primary context), after which this entry point must not
 *    be called again in that process.
 *  - Calls no allocating routine (no cudaMalloc / cudaFree).
 */
#define SDPA_NOALLOC_SCRATCH_BYTES (16u << 20)
sdpa_status_t sdpa_bwd_noalloc(const sdpa_shape* shape, const void* q, const void* k,
                               const void* v, const void* o, const void* dout,
                               const float* lse, const sdpa_bias_desc* bias,
                               const sdpa_mask_spec* mask, float scale, void* dq,
                               void* dk, void* dv, int32_t deterministic, void* stream);

/*
 * Backward plus the gradient of the additive bias, for training a learnable
 * bias (catie-aq/flashT5 README: "Full attention biases" and "T5-like
 * relative position encoding biases").  The scores are linear in the bias,
 * so with dS = P (dP - D) as in sdpa_bwd:
 *   DENSE: dbias[b, h, i, j] = sum of dS[b', h', i, j] over the (b', h')
 *          that read bias[b, h, i, j]: dS itself for a full-shape bias,
 *          summed over batch and / or heads where stride_b / stride_h = 0.
 *          dbias is float32 with the bias's own strides (a padded bias
 *          gives an equally padded dbias; padding is not written), 16-byte
 *          aligned.  The bias's kept indices must nest b > h > i without
 *          overlap (stride_i >= L, stride_h >= L stride_i, stride_b >= Hq
 *          stride_h, skipping broadcast indices), else SDPA_ERR_UNSUPPORTED.
 *          Masked (i, j), and keys of tiles the mask skips, get 0.
 *   T5:    dbias[k * Hq + h] = sum of dS[b, h, i, j] over every (b, i, j)
 *          with bucket(j - i) = k: float32 [num_buckets, Hq] like the table,
 *          16-byte aligned.
 *   ALIBI: dbias[h] = -sum of |j - i| dS[b, h, i, j] over every (b, i, j):
 *          the gradient of the slopes, float32 [Hq], 16-byte aligned.
 *   REL:   dbias[(r + L - 1) * Hq + h] = sum of dS[b, h, i, i + r] over every
 *          (b, i): float32 [2L - 1, Hq] like the table, 16-byte aligned.
 *   NONE:  SDPA_ERR_UNSUPPORTED.
 * dq, dk, dv as sdpa_bwd.  Deterministic: every sum is taken in one fixed
 * order, so repeated calls give identical bits.
 * workspace: at least sdpa_bwd_bias_grad_workspace_size(shape, bias) bytes,
 * 256-byte aligned, contents ignored on entry.  A broadcast dense bias
 * stages an fp32 copy of dS there (B * Hq * L rows of L floats padded to a
 * multiple of 8) and reduces it; T5, ALiBi and REL stage no dS.  T5: the
 * dQ kernel sums dS per bucket and warp over each query tile's key tiles,
 * 8 * num_buckets floats per (batch, head, query tile); ALiBi: it sums
 * |j - i| dS per warp, 8 floats per (batch, head, query tile, key tile);
 * REL: it sums dS along the distances j - i per warp, 1280 floats per
 * (batch, head, query tile, key tile), folded in fixed order.  A
 * full-shape dense bias stages nothing.  dbias must not overlap any other
 * argument.
 */
size_t sdpa_bwd_bias_grad_workspace_size(const sdpa_shape* shape, const sdpa_bias_desc* bias);
sdpa_status_t sdpa_bwd_bias_grad(const sdpa_shape* shape, const void* q, const void* k,
                                 const void* v, const void* o, const void* dout,
                                 const float* lse, const sdpa_bias_desc* bias,
                                 const sdpa_mask_spec* mask, float scale, void* dq, void* dk,
                                 void* dv, float* dbias, int32_t deterministic, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * T5 bucket ids of n signed distances rel[i] = key_pos - query_pos, computed
 * by the same device function the kernels use (device pointers, int32).
 * Exported so the bucketing can be checked bit-exactly on its own.
 */
sdpa_status_t sdpa_t5_bucket(const int32_t* rel, int32_t* out, int64_t n,
                             int32_t num_buckets, int32_t max_distance,
                             int32_t bidirectional, void* stream);

/*
 * y[i] = 2^x[i] by the kernels' FMA-pipe exponential (Cody-Waite reduction
 * and a fitted cubic; relative error below 1.2e-4 for -125 <= x <= 125),
 * device pointers, float32.  Exported so the approximation can be checked
 * against exp2 on its own.
 */
sdpa_status_t sdpa_exp2_fma(const float* x, float* y, int64_t n, void* stream);

/*
 * Synchronises `stream`, then returns and clears the sticky device status of
 * the current device: SDPA_OK; SDPA_ERR_TIMEOUT if any kernel's bounded wait
 * ran out since the last call; SDPA_ERR_UNSUPPORTED if a kernel found its
 * shared memory not 1024-byte aligned and returned without computing;
 * SDPA_ERR_CUDA if the reads fail.
 */
sdpa_status_t sdpa_read_device_status(void* stream);

/*
 * Sets the time limit of every bounded in-kernel wait, in nanoseconds
 * (default 2e9; values below 1000 are raised to 1000).  Host-side setting,
 * read at each launch.
 */
void sdpa_set_wait_limit_ns(uint64_t ns);

/*
 * Launches one CTA that waits on a barrier nothing ever completes, under the
 * current wait limit, so the timeout path can be exercised without faulting
 * or hanging the GPU.  Expect sdpa_read_device_status() == SDPA_ERR_TIMEOUT
 * afterwards.
 */
sdpa_status_t sdpa_debug_wait_timeout(void* stream);

/*
 * FIRE relative-position bias as a REL table.  The catie-aq/flashT5 README
 * names FIRE among the positional schemes it means to support and gives no
 * formula; this is the bias of Li et al. 2023 ("Functional Interpolation for
 * Relative Positions Improves Long Context Transformers"):
 *   bias[h, i, j] = f_h(psi(|i - j|) / psi(threshold)),  psi(t) = log(c t + 1),
 *   f(x) = w2 relu(w1 x + b1) + b2  (one hidden layer of `width` units).
 * The paper divides by psi(max(threshold, i)); with threshold >= Lq - 1 (a
 * requirement here, else SDPA_ERR_UNSUPPORTED) that is psi(threshold) on
 * every row, so the bias depends on the distance alone; keys after the
 * query take the same function of |i - j|.  All pointers are device float32:
 * w1, b1 [width], w2 [heads][width], b2 [heads]; 1 <= width <= 1024,
 * 1 <= heads <= 65535, c > 0.  Arithmetic in float32.
 */
typedef struct sdpa_fire {
  const float* w1;
  const float* b1;
  const float* w2;
  const float* b2;
  float c;
  float threshold;
  int32_t width;
  int32_t heads;
} sdpa_fire;

/* table [Lq + Lk - 1][heads] (device, caller-owned): the REL table of FIRE. */
sdpa_status_t sdpa_fire_table(const sdpa_fire* fire, int64_t Lq, int64_t Lk, float* table,
                              void* stream);

/* Bytes of device workspace sdpa_fire_backward needs (0 for bad arguments). */
size_t sdpa_fire_backward_workspace_size(const sdpa_fire* fire, int64_t Lq, int64_t Lk);

/*
 * Gradients of sum(d_table * table) with respect to FIRE's parameters, from
 * the gradient of its table (sdpa_bwd_bias_grad with a REL bias returns
 * it): d_w1, d_b1 [width], d_w2 [heads][width], d_b2 [heads], d_c_threshold
 * [2] = (d/dc, d/dthreshold); all device float32, written in full.  Every
 * output is a sum over the table rows in a fixed order (deterministic).
 */
sdpa_status_t sdpa_fire_backward(const sdpa_fire* fire, int64_t Lq, int64_t Lk,
                                 const float* d_table, float* d_w1, float* d_b1, float* d_w2,
                                 float* d_b2, float* d_c_threshold, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Static English text for a status code. */
const char* sdpa_status_string(sdpa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_B200_SDPA_H */
