/*
 * fa.h — C ABI of libfa.so: fused exact-attention forward on B200 (sm_100a),
 * BF16 and FP8-e4m3 (for Q Kᵀ), its BF16 backward pass, and the Hadamard
 * rotate-and-quantise step that prepares FP8 queries and keys.
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" must point to memory of the CUDA device that is
 *    current on the calling thread; the caller allocates and owns every buffer.
 *    The library allocates no device memory.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). All work is
 *    enqueued on it; nothing synchronises the host.
 *  - Argument errors are returned before anything is enqueued. A failed launch
 *    returns FA_ERR_CUDA. A device-side failure (a bounded wait that ran out)
 *    is recorded on the device and read with fa_device_status().
 *  - Tensors are dense and row-major ("contiguous"), with the layouts stated.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, size < 1, bad scale, workspace too small */
  FA_ERR_UNSUPPORTED = 2, /* head dimension / dtype combination not built */
  FA_ERR_ALIGNMENT = 3,   /* a pointer is not aligned as required */
  FA_ERR_CUDA = 4,        /* a CUDA call or a launch failed */
  FA_ERR_TIMEOUT = 5      /* (device status only) a bounded wait inside a kernel ran out */
} fa_status;

typedef enum {
  FA_BF16 = 0,       /* Q and K are bf16 */
  FA_E4M3 = 1,       /* Q and K are e4m3 codes (one byte each) with per-tensor descales */
  FA_E4M3_BLOCK = 2  /* e4m3 codes with one descale per 128-row block of a head */
} fa_dtype;

/*
 * fa_fwd — exact attention forward with per-row log-sum-exp.
 *
 * Defined by: "Flash Attention" glossary page, paragraphs 1-2 (the output equals
 * standard attention softmax(scale Q Kᵀ) V; the N x N matrix is never written to
 * HBM, tiles are processed on chip with an online, numerically stable softmax),
 * and "FlashAttention-3 (PT)", section "FlashAttention e FlashAttention-2"
 * (tiling; matmul, softmax and matmul fused in one kernel). For every batch b,
 * head h and query row i:
 *   O[b,h,i,:] = sum_j w_ij V[b,h,j,:],  w_ij = exp(z_ij) / sum_j' exp(z_ij'),
 *   z_ij = scale * Q[b,h,i,:] . K[b,h,j,:],   LSE[b,h,i] = ln sum_j exp(z_ij),
 * with j over 0..N-1, or over 0..i when `causal` != 0 (square mask, top-left).
 *
 * q, k    device, [B][H][N][d]; bf16 when qk_dtype = FA_BF16, e4m3 codes when
 *         FA_E4M3 (then Q = dq * decode(q), K = dk * decode(k)). 16-byte aligned.
 * v       device, bf16 [B][H][N][d], 16-byte aligned.
 * o       device, bf16 [B][H][N][d] output (round to nearest even), 16-byte aligned.
 * lse     device, fp32 [B][H][N] output (natural log), 4-byte aligned; may be NULL.
 * B, H, N >= 1; d in {64, 128, 256} for FA_BF16, {128, 256} for FA_E4M3.
 * scale   finite and > 0 (usually 1/sqrt(d)).
 * descale_qk  device fp32: for FA_E4M3 two values {dq, dk} (as written by
 *         fa_hadamard_quant); for FA_E4M3_BLOCK the B*H*ceil(N/128) query-block
 *         descales followed by the B*H*ceil(N/128) key-block descales, each
 *         [B][H][block] (as written by fa_hadamard_quant_blocks); ignored (may be
 *         NULL) for FA_BF16.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                 int d, int causal, float scale, fa_dtype qk_dtype, const float* descale_qk, void* stream);

/*
 * fa_fwd_splitkv — attention of Nq queries over Nk keys per head (decode- and
 * chunk-shaped problems: few queries, long key sequences), with the keys split
 * into n_split blocks that separate CTAs process in parallel, then merged.
 *
 * Defined by: the same output as fa_fwd (standard attention; "Flash Attention"
 * glossary page, paragraphs 1-2), for a query block that is the last Nq
 * positions of the key sequence. The split follows the glossary page's second
 * paragraph: the online softmax accumulates results over blocks of keys; here
 * the blocks are computed at once and combined by their LSEs (fa_lse_merge).
 * FlashDecoding++ ("FlashAttention-3 (PT)", references) is the pages' title for
 * this decode setting; the pages give no algorithm for it. For query row i:
 *   key j is visible iff j < Nk and (causal == 0 or j <= i + (Nk - Nq)).
 *
 * q       device, [B][H][Nq][d] (bf16, or e4m3 codes for FA_E4M3), 16-byte aligned.
 * k, v    device, [B][H][Nk][d] (k: bf16 or e4m3 codes; v: bf16), 16-byte aligned.
 * o       device, bf16 [B][H][Nq][d] output; lse fp32 [B][H][Nq] (natural log) or NULL.
 * B, H, Nq, Nk >= 1; causal requires Nq <= Nk. d, scale, qk_dtype: as fa_fwd;
 *         descale_qk as fa_fwd, with FA_E4M3_BLOCK holding B*H*ceil(Nq/128) query
 *         blocks then B*H*ceil(Nk/128) key blocks.
 * n_split 1 = no split (no workspace; the same kernel as fa_fwd); >= 2 = that many
 *         blocks of ceil(ceil(Nk/128)/n_split) key tiles of 128 keys (the last ones
 *         may be empty); 0 = automatic: with fewer query blocks (of 128 or 256
 *         rows) than SMs, fa_fwd_splitkv_splits(B, H, Nq, Nk, d) blocks for every
 *         query block; else, without causal masking, when the last round of
 *         query blocks over the SMs (one CTA per SM) is at most half full and a
 *         head has at least 4 key tiles, each block of that round as 2-4 pieces
 *         over disjoint key tiles, merged by their LSEs inside the kernel (the
 *         result does not depend on the order the pieces finish in); else no
 *         split.
 * workspace  device, >= fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, n_split)
 *         bytes, 256-byte aligned, owned by the caller (may be NULL if that is 0);
 *         overwritten; its contents before the call do not matter. Calls that
 *         overlap on the GPU must not share it.
 * Errors: FA_ERR_INVALID_ARG (also: workspace missing or too small),
 *         FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                         int Nk, int d, int causal, float scale, fa_dtype qk_dtype, const float* descale_qk,
                         int n_split, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of fa_fwd_splitkv for these sizes (n_split = 0: the automatic
 * schedule on the current device); 0 when no workspace is needed or on bad sizes. */
size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int n_split);

/* The split count fa_fwd_splitkv uses for n_split = 0 on the current device: the
 * count that gives the fewest key-tile steps on the busiest SM (one CTA per SM),
 * at least 1. */
int fa_fwd_splitkv_splits(int B, int H, int Nq, int Nk, int d);

/*
 * fa_fwd_partial — the per-block results of fa_fwd_splitkv, without the merge:
 * for block s (keys of tiles s*T .. s*T+T-1, T = ceil(ceil(Nk/128)/n_split)), the
 * output normalised over that block's visible keys and its LSE. Blocks computed
 * by separate calls (for example over key chunks that arrive one at a time from
 * other devices, as in ring attention: "Flash Attention" glossary page, fourth
 * paragraph) combine with fa_lse_merge.
 *
 * o_part    device, fp32 [n_split][B][H][Nq][d], 16-byte aligned.
 * lse_part  device, fp32 [n_split][B][H][Nq] (natural log), 4-byte aligned. A row
 *           with no visible key in a block gets O = 0 and LSE = -inf there.
 * Other arguments as fa_fwd_splitkv (n_split >= 1).
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int H,
                         int Nq, int Nk, int d, int causal, float scale, fa_dtype qk_dtype, const float* descale_qk,
                         int n_split, void* stream);

/*
 * fa_lse_merge — combine results over disjoint blocks of keys into the result over
 * their union. With M = max_s LSE_s and w_s = exp(LSE_s - M) per row:
 *   O = sum_s w_s O_s / sum_s w_s  (bf16, round to nearest even),
 *   LSE = M + ln sum_s w_s;        rows with every LSE_s = -inf get O = 0, LSE = -inf.
 * Defined by: "Flash Attention" glossary page, second paragraph (the online
 * softmax's rescale of partial results), applied to whole partial results.
 *
 * o_part    device, fp32 [n_part][rows][d], 16-byte aligned; lse_part fp32 [n_part][rows].
 * o         device, bf16 [rows][d], 16-byte aligned; lse fp32 [rows] or NULL.
 * n_part >= 1; rows >= 1; d in {64, 128, 256}.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_lse_merge(const float* o_part, const float* lse_part, int n_part, int64_t rows, int d, void* o,
                       float* lse, void* stream);

/*
 * fa_bwd — gradients of a loss through exact attention: given dO = dLoss/dO for
 * O = softmax(scale Q Kᵀ) V (square heads, as fa_fwd computes it), return
 *   dV = Pᵀ dO,  dS = P ∘ (dO Vᵀ - D),  D_i = dO_i · O_i,
 *   dQ = scale dS K,  dK = scale dSᵀ Q,
 * per batch and head, with P the attention probabilities (causal: key j hidden
 * from query i when j > i). The pages name training with the method
 * ("FlashAttention-3 (PT)", opening paragraph and section "Desempenho e
 * importância") but give no backward algorithm: this is the chain rule through
 * the definition fa_fwd documents. P is recomputed on chip from Q, K and the
 * forward's LSE, so no N x N matrix is written ("Flash Attention" glossary page,
 * second paragraph). D_i uses the given O, as the forward returned it.
 *
 * q, k, v, o, dout   device, bf16 [B][H][N][d], 16-byte aligned (o: fa_fwd's output).
 * lse                device, fp32 [B][H][N]: fa_fwd's LSE (natural log), 4-byte aligned.
 * dq, dk, dv         device, bf16 [B][H][N][d] outputs (round to nearest even), 16-byte aligned.
 * B, H, N >= 1; d in {64, 128} (d = 256 returns FA_ERR_UNSUPPORTED: dK and dV of a
 * 128-key tile would need all of a CTA's tensor memory); scale finite and > 0.
 * workspace          device, >= fa_bwd_workspace_bytes(B, H, N, d) bytes, 256-byte
 *                    aligned: the fp32 dQ accumulator and the per-row D and LSE.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int N, int d, int causal, float scale,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace fa_hadamard_quant and fa_hadamard_quant_multi need (an amax
 * word and a grid-barrier counter per tensor, padded). */
#define FA_QUANT_WORKSPACE_BYTES 256

/*
 * fa_fwd_fp8_qrot — e4m3 attention forward with Q rotated and quantised inside
 * the attention kernel: Q is given in bf16, and each 128-row query tile is
 * rotated and quantised to e4m3 with its own scale in shared memory, right
 * after it is loaded and before its first Q Kᵀ. K is given as e4m3 codes with
 * one descale per 128-row block (fa_hadamard_quant_blocks, with the same
 * rotation). The result is that of fa_fwd with qk_dtype = FA_E4M3_BLOCK on Q
 * quantised by fa_hadamard_quant_blocks, without the separate pass over Q.
 *
 * Defined by: "FlashAttention-3 (PT)", section "Inovações técnicas",
 * subsection 3 ("Baixa precisão (FP8)"), steps 1-4, with one scale per block of
 * 128 rows; the attention itself as for fa_fwd.
 *
 * q          device, bf16 [B][H][N][d], 16-byte aligned.
 * k8         device, e4m3 codes [B][H][N][d] (uint8), 16-byte aligned.
 * v          device, bf16 [B][H][N][d], 16-byte aligned.
 * o, lse     as fa_fwd (lse may be NULL).
 * d          128 only (FA_ERR_UNSUPPORTED otherwise).
 * dk_blocks  device, fp32 [B][H][ceil(N/128)]: K's block descales.
 * rotate     1: x' = x diag(signs) H_128 / sqrt(128) before quantising (as K was);
 *            0: quantise only.
 * signs      device, 128 fp32 values +-1 (16-byte aligned), or NULL for none.
 * dq_blocks_out  device, fp32 [B][H][ceil(N/128)] receiving each query
 *            block's descale (amax / 448), or NULL.
 * Errors: as fa_fwd.
 */
fa_status fa_fwd_fp8_qrot(const void* q, const void* k8, const void* v, void* o, float* lse, int B, int H, int N,
                          int d, int causal, float scale, const float* dk_blocks, int rotate, const float* signs,
                          float* dq_blocks_out, void* stream);

/*
 * fa_hadamard_quant — rotate (optionally) and quantise one tensor to e4m3 with a
 * single scale.
 *
 * Defined by: "FlashAttention-3 (PT)", section "Inovações técnicas", subsection 3
 * ("Baixa precisão (FP8)"), steps 1-4: queries and keys are multiplied by a random
 * orthogonal (Hadamard) matrix, which spreads outlier coordinates, then quantised
 * to FP8; Q Kᵀ is unchanged by the rotation. Per row r:
 *   x'[r,:] = x[r,:] diag(signs) H_d / sqrt(d)   (H_d: Sylvester Hadamard)  if rotate,
 *   x'[r,:] = x[r,:]                                                       otherwise;
 *   amax = max |x'| over the whole tensor;  descale = amax / 448 (1 if amax = 0);
 *   out[r,c] = e4m3(x'[r,c] * 448 / amax), round to nearest even, saturating.
 *
 * x           device, bf16 [rows][d], 16-byte aligned (e.g. [B][H][N][d], rows = B*H*N);
 *             may be NULL when rows = 0.
 * out         device, e4m3 codes [rows][d], 16-byte aligned; may be NULL when rows = 0.
 * descale_out device, one fp32 (written in the second pass, after the grid-wide amax).
 * rows        0 .. 2^31 - 4097 (TMA tile coordinates are 32-bit; a larger bf16
 *             tensor would not fit in device memory);  d in {64, 128, 256}.
 * rotate      0 = quantise only, 1 = rotate first.
 * signs       device, d fp32 values +-1 (16-byte aligned), or NULL for no sign flips.
 * workspace   device scratch of >= FA_QUANT_WORKSPACE_BYTES bytes, 16-byte aligned,
 *             owned by the caller; its contents are overwritten. Calls that overlap on
 *             the GPU must not share one workspace.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_hadamard_quant(const void* x, void* out, float* descale_out, int64_t rows, int d, int rotate,
                            const float* signs, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_quant_v_transposed — V's e4m3 codes with one scale per tensor, written with
 * the keys along the contiguous dimension.
 *
 * Defined by: "FlashAttention-3 (PT)", section "Inovações técnicas", subsection 3
 * (FP8 operands quantised with a scale; only Q and K are rotated). The pages give
 * neither V's scale granularity nor its layout; this entry takes one scale per
 * tensor and no rotation:
 *   amax = max |v| over the tensor;  descale_out[0] = amax / 448 (1 if amax = 0);
 *   out_t[bh][c][n] = e4m3(fl(v[bh][n][c] * fl(448 / amax)))  (RNE, saturating),
 * the same codes fa_hadamard_quant gives with rotate = 0, transposed per head.
 *
 * v          device bf16 [BH][N][d] (B and H folded), 16-byte aligned.
 * out_t      device e4m3 codes [BH][d][N], 16-byte aligned.
 * descale_out device fp32, 1 value.
 * BH in 1..65535, N >= 1, d in {64, 128, 256}; BH * N rows at most 2^31 - 4096.
 * workspace  device, >= FA_QUANT_WORKSPACE_BYTES, 16-byte aligned (the amax word;
 *            zeroed here). Calls that overlap on the GPU must not share it.
 * Two launches on `stream` (the amax, then the codes).
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_quant_v_transposed(const void* v, void* out_t, float* descale_out, int BH, int N, int d,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_hadamard_quant_multi — fa_hadamard_quant for up to 8 tensors of one shape
 * (for example Q and K) in one launch, each with its own scale: the same codes
 * and descales as one call per tensor, with one grid-wide barrier in place of one
 * per tensor.
 *
 * Defined by: as fa_hadamard_quant.
 * xs, outs  host arrays of `ntensors` device pointers: bf16 inputs [rows][d] and
 *           e4m3 outputs [rows][d], each 16-byte aligned (may be NULL if rows = 0).
 * descales  device, ntensors fp32 (tensor i's descale at descales[i]).
 * ntensors  1..8. rows, d, rotate, signs, workspace: as fa_hadamard_quant (the
 *           workspace holds the amax words and the barrier counter).
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_hadamard_quant_multi(const void* const* xs, void* const* outs, float* descales, int ntensors,
                                  int64_t rows, int d, int rotate, const float* signs, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * fa_hadamard_quant_blocks — rotate (optionally) and quantise one tensor to e4m3
 * with one scale per block of 128 consecutive rows of each head (the attention
 * kernel's query and key tiles), in one pass over the input.
 *
 * Defined by: the same steps as fa_hadamard_quant ("FlashAttention-3 (PT)",
 * section "Inovações técnicas", subsection 3), with the amax taken per block
 * instead of per tensor; the pages give no block size. Per block b of a head (rows
 * 128b .. min(N, 128b+128)):
 *   amax_b = max |x'| over the block;  descales[head][b] = amax_b / 448 (1 if 0);
 *   out = e4m3(x' * 448 / amax_b), round to nearest even, saturating.
 *
 * x         device, bf16 [BH][N][d], 16-byte aligned.
 * out       device, e4m3 codes [BH][N][d], 16-byte aligned.
 * descales  device, fp32 [BH][ceil(N/128)], 4-byte aligned.
 * BH, N >= 1; d in {64, 128, 256}; rotate, signs: as fa_hadamard_quant.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_hadamard_quant_blocks(const void* x, void* out, float* descales, int BH, int N, int d, int rotate,
                                   const float* signs, void* stream);

/*
 * fa_hadamard_quant_noalloc — fa_hadamard_quant for callers that cannot allocate
 * device memory, for up to 64 tensors of one shape (e.g. Q and K) per call.
 *
 * No counterpart in the pages: this is a service entry point of this library.
 * Some callers cannot call cudaMalloc or hand over a workspace: code that owns
 * no device allocator (a plugin inside an application that manages all device
 * memory itself), or code that must not trigger the implicit device-wide
 * synchronisation an allocation can cause. This entry point needs no workspace:
 * the scratch (one 4-byte amax word per tensor and 8 grid-barrier counters) is
 * a 288-byte array inside the library, allocated when the library is loaded and
 * held by every device that loads it until the process exits. Results are
 * identical to calling fa_hadamard_quant once per tensor.
 *
 * xs, outs   host arrays of `ntensors` device pointers: bf16 inputs [rows][d] and
 *            e4m3 outputs [rows][d], each 16-byte aligned (may be NULL if rows = 0).
 * descales   device, ntensors fp32 (descale of tensor i at descales[i]).
 * ntensors   1..64; more is rejected with FA_ERR_INVALID_ARG (the array holds 64 amax words).
 * rows, d, rotate, signs: as for fa_hadamard_quant, shared by all tensors.
 * The first call on a device looks up the array's device address (a one-time
 * set-up per device, with that device current); make that first call before any
 * stream capture. Every call zeroes and reuses the same array, so calls that
 * overlap on the GPU (other streams, other host threads) race and must be
 * serialised by the caller.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA.
 */
fa_status fa_hadamard_quant_noalloc(const void* const* xs, void* const* outs, float* descales, int ntensors,
                                    int64_t rows, int d, int rotate, const float* signs, void* stream);

/* Human-readable name of a status code (static string). */
const char* fa_status_string(fa_status s);

/*
 * fa_device_status — read and clear the device-side status of the current
 * device. Synchronises the device first. *code receives FA_OK or FA_ERR_TIMEOUT,
 * *site an internal wait-site number and *block the CTA index that recorded it;
 * any output pointer may be NULL. Returns FA_ERR_CUDA if the read itself failed.
 */
fa_status fa_device_status(int* code, unsigned int* site, unsigned int* block);

/* ABI version of this header: 6 (1, plus the split-key, partial and merge calls in 2,
 * plus per-block e4m3 scales in 3, plus the backward pass in 4, plus
 * fa_fwd_fp8_qrot in 5, plus fa_quant_v_transposed in 6). */
int fa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
