/*
 * bitlinear.h — C ABI of the B200 (sm_100a) BitNet b1.58 BitLinear forward.
 *
 * The operations follow the blog post "BitNet b1.58 — quantização ternária,
 * BitLinear, Zero-GEMM" (BLOG below) and the API names of "Arquitetura
 * Hibrida Multimodal para bitnet.cpp", section utils/ — bit_layers.py
 * (quantise_weights_ternary, quantise_activations_8bit, BitLinear,
 * ReLUSquared).
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  * Tensors are row-major and contiguous. Activations A are [M, K]
 *    (tokens × in-features); weights W are [N, K] (out × in, the nn.Linear
 *    layout); outputs Y are [M, N]. The layer computes Y = f(A · Wᵀ).
 *  * Every pointer argument, unless stated otherwise, is a DEVICE pointer to
 *    memory the caller owns. The library never allocates, frees or keeps
 *    pointers after the call returns. Scratch memory ("workspace") is passed
 *    in by the caller; its size comes from the matching *_workspace_bytes().
 *    For bl_zero_gemm, bl_linear_q, bl_linear and bl_ffn_relu2 part of that
 *    size is optional: with more than 32 tokens and too few output tiles to
 *    fill half of the SMs, the tensor-core contraction splits K into up to 4
 *    ranges whose INT32 partials go there before one summing pass; a smaller
 *    workspace (down to the quantised tokens and row sums) gives the same
 *    results unsplit.
 *  * Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and makes no host synchronisation. Scales
 *    (γ, γ_A) are passed by device pointer for the same reason.
 *  * Pointers must be 16-byte aligned. K must be a positive multiple of 64
 *    and at most BL_MAX_K (the same holds for the FFN hidden size H);
 *    M, N ≥ 0 (M == 0 or N == 0 is a no-op returning BL_OK). eps must be
 *    finite and > 0. NaN/Inf inputs are outside the contract (not checked).
 *  * BL_MAX_K = 2^22 keeps every INT32 sum exact: |Σ_k A_q·W_q| ≤ 127·K
 *    < 2^31, and so do the kernels' internal partial sums (the decode GEMV
 *    keeps sums scaled by up to 64 per thread).
 *  * Errors are returned, never thrown or aborted: argument errors are found
 *    on the host before any launch (nothing is launched then); launch errors
 *    map to BL_ERR_CUDA. Device-side waits are bounded: a wait that gives up
 *    raises a per-device error flag, read (and cleared) by
 *    bl_check_device_error().
 *  * The device must be sm_100 (B200); otherwise BL_ERR_UNSUPPORTED.
 *
 * Packed ternary weight format (this library's; the BLOG, section "Como o
 * BitNet quebra o Memory Wall...", fixes only "2 bits per weight"):
 *  * code c = w + 1 ∈ {0, 1, 2} for w ∈ {-1, 0, +1}; 3 is never written;
 *  * a row of K weights is K/16 little-endian 32-bit words (K/4 bytes),
 *    rows are contiguous: the packed matrix is [N, K/4] bytes;
 *  * within word g of a row, weight k = 16·g + 4·j + i (i, j ∈ 0..3) sits in
 *    bits 8·i + 2·j and 8·i + 2·j + 1.
 *  So (word >> 2·j) & 0x03030303 holds the codes of weights 16g+4j .. 16g+4j+3
 *  as four bytes in natural order.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BL_OK = 0,
  BL_ERR_INVALID_ARG = 1, /* null pointer, bad eps, bad flag or dtype value */
  BL_ERR_SHAPE = 2,       /* negative size, K not a positive multiple of 64,
                             size too large for the kernels' index types */
  BL_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  BL_ERR_DTYPE = 4,       /* dtype not allowed for this argument */
  BL_ERR_CUDA = 5,        /* a CUDA runtime/driver call or launch failed */
  BL_ERR_TIMEOUT = 6,     /* a device-side bounded wait gave up */
  BL_ERR_UNSUPPORTED = 7, /* current device is not sm_100 */
  BL_ERR_WORKSPACE = 8    /* workspace missing or smaller than required */
} bl_status;

typedef enum { BL_F32 = 0, BL_BF16 = 1 } bl_dtype;

/* Largest K (and FFN hidden size H) any entry point accepts. */
#define BL_MAX_K 4194304

/* cudaStream_t-compatible handle (cudaStream_t is struct CUstream_st*). */
typedef struct CUstream_st* bl_stream_t;

/* Flags for the *_ex entry points. */
enum {
  /* Launch with programmatic dependent launch: the kernel streams its packed
   * weights into shared memory BEFORE waiting for the previous kernel on the
   * stream, and lets the next kernel start early. Only valid when the weight
   * buffer was NOT written by the kernel immediately preceding this call on
   * `stream` (true for a decode chain over static weights). Activations and
   * outputs are still ordered after the previous kernel. Above
   * bl_gemv_max_tokens() tokens the flag makes the activation quantiser
   * launch early too (it waits for the previous kernel before touching
   * memory), so the contraction's CTAs can stream their weights during the
   * previous call. */
  BL_FLAG_PDL = 1,
  /* bl_linear_radix3 / bl_linear_lut only: Y is the raw INT32
   * accumulator [M, N]. */
  BL_FLAG_RAW_I32 = 2
};

/* Human-readable name of a status code (static string, never NULL). */
const char* bl_status_string(bl_status s);

/* Library ABI version (major*100 + minor). */
int bl_version(void);

/* Number of decoded tokens up to which bl_linear uses the fused GEMV path. */
int bl_gemv_max_tokens(void);

/* Which kernel contracts M int8 tokens with an N × K packed matrix, on a
 * device with `sms` SMs, when the call's workspace has split_ws_bytes of room
 * for K-split partials (the optional part of the *_workspace_bytes() sizes):
 *   0  the fused GEMV: M ≤ bl_gemv_max_tokens() and one weight row plus the
 *      M token rows fit a CTA's shared memory (K ≤ 37,376 at 1 token, 28,096
 *      at 2, 22,464 at 3, 18,624 at 4); longer rows take path 1;
 *   1  the warp-level int8 MMA kernel (5 ≤ M ≤ 32, and 33–64 tokens when the
 *      tensor-core tiles, times their K ranges, would fill under half of the
 *      SMs);
 *   2  tensor-core tiles, K unsplit;
 *   3  tensor-core tiles with K split into ranges.
 * -1 for a non-positive size or K not a multiple of 64. Host only: reads no
 * device state and launches nothing. */
int bl_contraction_path(int64_t M, int64_t N, int64_t K, int sms, size_t split_ws_bytes);

/* ---------------------------------------------------------------------------
 * bl_quant_weights — quantise_weights_ternary.
 * BLOG, section "Por que 1,58 bits por peso e qual a matemática da
 * ternarização?": γ = (1/(N·K)) Σ|W_ij| over the whole matrix;
 * W_q = Round(Clip(W / (γ+ε), -1, 1)) ∈ {-1, 0, +1}, Round = half-to-even.
 *   W         [N, K] fp32 or bf16 (w_dtype), device.
 *   W_packed  [N, K/4] bytes, device, written in the packed format above.
 *   gamma     1 fp32, device, written with γ (sum in double, rounded once).
 *   workspace ≥ bl_quant_weights_workspace_bytes(N, K) bytes, device.
 * The code decision equals the fp32 division W ÷ (γ+ε) followed by
 * round-half-to-even, exactly.
 */
size_t bl_quant_weights_workspace_bytes(int64_t N, int64_t K);
bl_status bl_quant_weights(const void* W, bl_dtype w_dtype, int64_t N, int64_t K,
                           float eps, uint8_t* W_packed, float* gamma,
                           void* workspace, size_t ws_bytes, bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * bl_quant_acts — quantise_activations_8bit.
 * BLOG, same section, activation paragraph: per token m,
 * γ_A[m] = max_k |A[m,k]|; A_q = Clip(Round(A · (127 / (γ_A+ε))), -128, 127),
 * taken in fp32 (127/(γ_A+ε) by IEEE division, then one fp32 product).
 *   A       [M, K] fp32 or bf16, device.
 *   A_q     [M, K] int8, device.
 *   gamma_A [M] fp32, device.
 *   rowsum  [M] int32, device, optional (NULL to skip): Σ_k A_q[m,k], the
 *           term the contraction kernels subtract to undo the +1 code
 *           offset; pass it on to bl_linear_q to save one pass.
 */
bl_status bl_quant_acts(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                        float eps, int8_t* A_q, float* gamma_A, int32_t* rowsum,
                        bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * bl_zero_gemm — the INT32 contraction alone.
 * BLOG, section "Como funciona a camada BitLinear e a eliminação de
 * multiplicações (Zero-GEMM)?": acc[m,n] = Σ_k W_q[n,k]·A_q[m,k] (add on +1,
 * subtract on -1, skip on 0), INT32 accumulation.
 *   A_q [M, K] int8; W_packed [N, K/4]; acc [M, N] int32 (all device).
 *   workspace ≥ bl_zero_gemm_workspace_bytes(M, K, N).
 */
size_t bl_zero_gemm_workspace_bytes(int64_t M, int64_t K, int64_t N);
bl_status bl_zero_gemm(const int8_t* A_q, int64_t M, int64_t K,
                       const uint8_t* W_packed, int64_t N, int32_t* acc,
                       void* workspace, size_t ws_bytes, bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * bl_linear_q — contraction + dequantisation from already-quantised tokens.
 * BLOG, Zero-GEMM section, last paragraph: Y = (A_q·W_qᵀ) · (γ_A·γ)/127, one
 * scalar per (token, matrix); with relu2 != 0, Y = max(Y, 0)² (ReLUSquared).
 * The scale is taken in fp32 as (γ_A[m]·γ)/127 (no ε, as the page writes it).
 *   A_q [M, K] int8; gamma_A [M] fp32; rowsum [M] int32 or NULL (then it is
 *   recomputed into the workspace); W_packed [N, K/4]; gamma 1 fp32;
 *   Y [M, N] fp32 or bf16 (y_dtype; bf16 rounds to nearest even).
 *   workspace ≥ bl_linear_q_workspace_bytes(M, K, N).
 */
size_t bl_linear_q_workspace_bytes(int64_t M, int64_t K, int64_t N);
bl_status bl_linear_q(const int8_t* A_q, const float* gamma_A,
                      const int32_t* rowsum, int64_t M, int64_t K,
                      const uint8_t* W_packed, const float* gamma, int64_t N,
                      int relu2, void* Y, bl_dtype y_dtype, void* workspace,
                      size_t ws_bytes, bl_stream_t stream);
/* bl_linear_q with `flags`: BL_FLAG_PDL as for bl_linear_ex (the kernel
 * before this call on `stream` does not write W_packed or gamma, so the
 * contraction may stream its weights before waiting for that kernel). */
bl_status bl_linear_q_ex(const int8_t* A_q, const float* gamma_A,
                         const int32_t* rowsum, int64_t M, int64_t K,
                         const uint8_t* W_packed, const float* gamma, int64_t N,
                         int relu2, void* Y, bl_dtype y_dtype, void* workspace,
                         size_t ws_bytes, unsigned flags, bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * bl_linear — BitLinear forward from float activations:
 * bl_quant_acts, bl_zero_gemm and the dequantisation of bl_linear_q in one
 * call. For M ≤ bl_gemv_max_tokens() it is a single fused GEMV launch (the
 * activation quantiser runs in the kernel prologue; no workspace needed) as
 * long as a weight row and the tokens fit one CTA's shared memory (K up to
 * 37,376 at 1 token, 18,624 at 4; bl_contraction_path says which); above
 * that, an activation-quantiser launch and one contraction launch:
 * warp-level int8 MMAs over all SMs for M ≤ 32, tensor-core (tcgen05) tiles
 * above. bl_linear_workspace_bytes follows the same rule. The contraction launches with programmatic dependent launch; it
 * reads no memory written by the kernel before it until that kernel has
 * completed, except that after this call's own quantiser it streams W_packed
 * early (the quantiser does not write it).
 *   A [M, K] fp32/bf16; W_packed [N, K/4]; gamma 1 fp32; Y [M, N] fp32/bf16.
 *   workspace ≥ bl_linear_workspace_bytes(M, K, N) (may be 0 → NULL ok).
 * bl_linear_ex adds `flags` (BL_FLAG_PDL).
 */
size_t bl_linear_workspace_bytes(int64_t M, int64_t K, int64_t N);
bl_status bl_linear(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                    const uint8_t* W_packed, const float* gamma, int64_t N,
                    float eps, int relu2, void* Y, bl_dtype y_dtype,
                    void* workspace, size_t ws_bytes, bl_stream_t stream);
bl_status bl_linear_ex(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                       const uint8_t* W_packed, const float* gamma, int64_t N,
                       float eps, int relu2, void* Y, bl_dtype y_dtype,
                       void* workspace, size_t ws_bytes, unsigned flags,
                       bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * Taps: the integers and scales the path decides on its way, written out
 * besides the normal result so that each can be compared, element by element,
 * with an independent implementation. Every pointer is a device buffer the
 * caller owns (16-byte aligned), or NULL to skip that tap.
 *   act_q      [M, K] int8  tokens the contraction used (AbsMax quantiser)
 *   act_gamma  [M]    fp32  γ_A per token
 *   act_rowsum [M]    int32 Σ_k A_q[m,k]
 *   acc_up     [M, H] int32 FFN only: up-projection accumulators
 *   req_q      [M, H] int8  FFN only: requantised ReLU² of the up-projection
 *   req_gamma  [M]    fp32  FFN only: γ_r per token
 *   req_rowsum [M]    int32 FFN only: Σ_n R_q[m,n]
 *   cta        On the fused GEMV path (bl_contraction_path() == 0) every CTA
 *              quantises the tokens for itself; the taps report the tokens
 *              of CTA `cta` (-1 or any value past the last CTA: the last one).
 * With more tokens the quantiser runs once in its own kernel and the taps are
 * copies of its outputs. The taps add device-to-device copies and one branch;
 * the computed results are those of the calls without taps. */
typedef struct {
  int8_t* act_q;
  float* act_gamma;
  int32_t* act_rowsum;
  int32_t* acc_up;
  int8_t* req_q;
  float* req_gamma;
  int32_t* req_rowsum;
  int32_t cta;
  int32_t reserved; /* must be 0 */
} bl_taps;

/* bl_linear_ex with taps (act_* only; the FFN taps must be NULL). */
bl_status bl_linear_taps(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                         const uint8_t* W_packed, const float* gamma, int64_t N,
                         float eps, int relu2, void* Y, bl_dtype y_dtype,
                         void* workspace, size_t ws_bytes, unsigned flags,
                         const bl_taps* taps, bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * bl_linear_noalloc — bl_linear for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment variant, not part of
 * the method.
 * Some callers own no device allocator on the path that runs the layer: a
 * plugin whose host runtime hands it only its input and output buffers and
 * owns every other byte of device memory, or a serving loop that must not
 * call cudaMalloc on its hot path (cudaMalloc may synchronise the device and
 * grows memory outside a fixed budget). This entry point takes the same
 * arguments as bl_linear minus the workspace and allocates nothing: the
 * scratch it needs off the fused GEMV path (bl_contraction_path() != 0: the int8
 * tokens, their scales and row sums: M·K + 8·M bytes, 256-byte aligned
 * pieces) lives in one fixed 4 MiB array inside the library. Every GPU that
 * loads the library holds that array until the process exits.
 *   * Sizes whose scratch exceeds 4 MiB (bl_linear_workspace_bytes(M, K, N) >
 *     4 MiB, e.g. M·K above about 4.1 million) are refused with
 *     BL_ERR_WORKSPACE before anything is launched; use bl_linear then.
 *   * The first call on a device looks up the array's device address (with
 *     that device current) and caches it together with the device's current
 *     context; make that first call before any stream capture. A call that
 *     finds a different context current (for example after
 *     cudaDeviceReset) looks the address up again, so it too must not be the
 *     first call inside a stream capture.
 *   * All calls on a device share the array, which keeps whatever the last
 *     call left in it. Nothing in it needs to start at zero (each call writes
 *     every byte it reads), but calls whose kernels overlap on the GPU (for
 *     example on two streams at once) race on it: order them on one stream.
 * Arguments, layouts and the other errors are those of bl_linear.
 */
bl_status bl_linear_noalloc(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                            const uint8_t* W_packed, const float* gamma, int64_t N,
                            float eps, int relu2, void* Y, bl_dtype y_dtype,
                            bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * bl_ffn_relu2 — ternary FFN block (BitLinear up → ReLU² → BitLinear down).
 * Composition of the BLOG formulas with ReLUSquared (bit_layers.py): per
 * token, h = dequantised up-projection (fp32), r = max(h,0)² (fp32), AbsMax
 * requantisation of r with the activation rule above (γ_r = max_n r), then
 * the down-projection dequantised with (γ_r·γ_down)/127.
 *   X [M, K] fp32/bf16; W_up [H, K/4]; gamma_up 1 fp32;
 *   W_down [K_out=K, H/4]; gamma_down 1 fp32; Y [M, K] fp32/bf16.
 *   H must be a positive multiple of 64.
 *   workspace ≥ bl_ffn_workspace_bytes(M, K, H).
 */
size_t bl_ffn_workspace_bytes(int64_t M, int64_t K, int64_t H);
bl_status bl_ffn_relu2(const void* X, bl_dtype x_dtype, int64_t M, int64_t K,
                       int64_t H, const uint8_t* W_up, const float* gamma_up,
                       const uint8_t* W_down, const float* gamma_down,
                       float eps, void* Y, bl_dtype y_dtype, void* workspace,
                       size_t ws_bytes, bl_stream_t stream);

/* bl_ffn_relu2 with flags: BL_FLAG_PDL launches the block's first kernel
 * (the up-projection GEMV, or the quantiser above bl_gemv_max_tokens()
 * tokens) with programmatic dependent launch, under the same contract as
 * bl_linear_ex: W_up and W_down were not written by the kernel preceding
 * this call on `stream`. */
bl_status bl_ffn_relu2_ex(const void* X, bl_dtype x_dtype, int64_t M, int64_t K,
                          int64_t H, const uint8_t* W_up, const float* gamma_up,
                          const uint8_t* W_down, const float* gamma_down, float eps,
                          void* Y, bl_dtype y_dtype, void* workspace, size_t ws_bytes,
                          unsigned flags, bl_stream_t stream);

/* bl_ffn_relu2 with taps: act_* report the quantised block input X_q, acc_up
 * the up-projection, req_* the requantised ReLU² tokens fed to the
 * down-projection (see bl_taps). */
bl_status bl_ffn_relu2_taps(const void* X, bl_dtype x_dtype, int64_t M,
                            int64_t K, int64_t H, const uint8_t* W_up,
                            const float* gamma_up, const uint8_t* W_down,
                            const float* gamma_down, float eps, void* Y,
                            bl_dtype y_dtype, void* workspace, size_t ws_bytes,
                            const bl_taps* taps, bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * Radix-3 weight storage for decode: five ternary weights per byte.
 * BLOG, section "Como o ecossistema bitnet.cpp acelera inferência em CPUs e
 * borda?": 3^5 = 243 ≤ 256 states, 1.60 bits per weight.
 * Layout (this library's): each row is cut into groups of five consecutive
 * weights, first weight most significant, b = Σ_i (w_i + 1)·3^(4-i) ∈
 * [0, 242]; the byte stored is q = ceil(256·b / 243) (b = floor(243·q/256));
 * weights past K count as 0; a row takes bl_radix3_row_bytes(K) =
 * 16·ceil(ceil(K/5)/16) bytes (padding groups hold all-zero weights).
 *   bl_pack_radix3: 2-bit packed [N, K/4] → radix-3 [N, row_bytes].
 *   bl_linear_radix3: bl_linear for M ≤ bl_gemv_max_tokens() tokens on
 *     radix-3 weights (one fused GEMV launch, same results as bl_linear);
 *     flags: BL_FLAG_PDL as for bl_linear_ex, BL_FLAG_RAW_I32 to write the
 *     INT32 accumulators instead (y_dtype ignored). M > 4, or K whose
 *     weight row and decode tables do not fit in one CTA's shared memory
 *     (K above 49,728 at 1 token, 30,080 at 2, 21,568 at 3, 16,768 at 4):
 *     BL_ERR_SHAPE. */
int64_t bl_radix3_row_bytes(int64_t K);
bl_status bl_pack_radix3(const uint8_t* W_packed, int64_t N, int64_t K, uint8_t* W_r3,
                         bl_stream_t stream);
bl_status bl_linear_radix3(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                           const uint8_t* W_r3, const float* gamma, int64_t N, float eps,
                           int relu2, void* Y, bl_dtype y_dtype, unsigned flags,
                           bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * Lookup-table decode (one token). BLOG, section "Como o ecossistema
 * bitnet.cpp acelera inferência em CPUs e borda?", figure "Fluxo de Execução
 * com Lookup Table (LUT-GEMM)": per block of 4 int8 activations a table of
 * the 81 signed sums of all ternary patterns; each group of 4 weights is one
 * index (27·d0 + 9·d1 + 3·d2 + d3, d = w + 1, first weight most significant:
 * 0 = all -1, 40 = all 0, 80 = all +1).
 *   bl_pack_lut_index: 2-bit packed [N, K/4] → index bytes [N, K/4]
 *     (byte g of a row indexes weights 4g .. 4g+3).
 *   bl_linear_lut: bl_linear for M = 1 on index bytes (tables of the token
 *     built in shared memory by every CTA; results equal bl_linear's);
 *     flags BL_FLAG_PDL, BL_FLAG_RAW_I32 as for bl_linear_radix3.
 *     M > 1, or K whose tables (K/4 · 41 int16) do not fit in a CTA's
 *     shared memory beside its weights (K above about 10,000): BL_ERR_SHAPE. */
bl_status bl_pack_lut_index(const uint8_t* W_packed, int64_t N, int64_t K, uint8_t* W_idx,
                            bl_stream_t stream);
bl_status bl_linear_lut(const void* A, bl_dtype a_dtype, int64_t M, int64_t K,
                        const uint8_t* W_idx, const float* gamma, int64_t N, float eps,
                        void* Y, bl_dtype y_dtype, unsigned flags, bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * Tensor-parallel FFN block: the per-rank steps of bl_ffn_relu2 when the
 * hidden dimension H is split over g ranks. The pages give no multi-GPU
 * design; this is the composition of the same formulas over a sharded H:
 * rank r holds rows [h0, h1) of W_up (column-parallel up-projection) and
 * columns [h0, h1) of W_down (row-parallel down-projection), with
 * H_r = h1 - h0 a positive multiple of 64 (W_down_r is then the contiguous
 * copy of bytes [h0/4, h1/4) of every packed row).
 *   1. bl_ffn_tp_up: AbsMax quantisation of X (identical on every rank),
 *      the shard's INT32 up-projection acc_up [M, H_r], γ_X [M], and
 *      rmax[m] = max over the shard of r = max(h, 0)² (fp32).
 *   2. the caller all-reduces rmax with MAX over the ranks: the result is
 *      γ_r of the unsharded block, bit for bit (a maximum is exact).
 *   3. bl_ffn_tp_down: requantisation of the shard's r with that γ_r and
 *      the shard's partial down-projection acc_down [M, K_out] (INT32).
 *   4. the caller all-reduces acc_down with SUM (INT32: exact, any order).
 *   5. bl_dequant_i32(acc_down, γ_r, γ_down) gives the block output, equal
 *      to bl_ffn_relu2's output bit for bit.
 * Workspaces come from the matching *_workspace_bytes(). */
size_t bl_ffn_tp_up_workspace_bytes(int64_t M, int64_t K);
bl_status bl_ffn_tp_up(const void* X, bl_dtype x_dtype, int64_t M, int64_t K, int64_t H_r,
                       const uint8_t* W_up_r, const float* gamma_up, float eps,
                       int32_t* acc_up, float* gamma_x, float* rmax, void* workspace,
                       size_t ws_bytes, bl_stream_t stream);
size_t bl_ffn_tp_down_workspace_bytes(int64_t M, int64_t H_r);
bl_status bl_ffn_tp_down(const int32_t* acc_up, const float* gamma_x, const float* gamma_up,
                         const float* gamma_r, int64_t M, int64_t H_r,
                         const uint8_t* W_down_r, int64_t K_out, float eps,
                         int32_t* acc_down, void* workspace, size_t ws_bytes,
                         bl_stream_t stream);

/* Y [M, N] = acc · ((γ_A[m]·γ)/127) in fp32 (relu2 != 0: max(Y, 0)²),
 * stored as fp32 or bf16 (round to nearest even): BLOG, Zero-GEMM section,
 * last paragraph, for INT32 accumulators computed elsewhere. */
bl_status bl_dequant_i32(const int32_t* acc, const float* gamma_A, const float* gamma,
                         int64_t M, int64_t N, int relu2, void* Y, bl_dtype y_dtype,
                         bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * STE backward (training). BLOG, Zero-GEMM section, paragraph after the
 * worked example: the gradient of the quantisation is taken as the identity
 * (∂W_q/∂W = 1) inside the valid range. With the forward Y = Â·Ŵᵀ,
 * Ŵ = γ·W_q and Â = (γ_A/127)·A_q:
 *   bl_ste_grad_input:  dA [M, K] = dY·Ŵ = γ·(dY·W_q)
 *   bl_ste_grad_weight: dW [N, K] = mask ⊙ (dYᵀ·Â), mask = 1 where the
 *                       forward's fp32 quotient W ÷ (γ+ε) lies in [-1, 1]
 *                       (W: the latent fp32/bf16 weights, [N, K]).
 * Arguments: dY [M, N] fp32 or bf16 (N a multiple of 8); W_packed, γ as for
 * bl_linear; A_q [M, K] int8 and γ_A [M] as bl_quant_acts returns them;
 * outputs fp32. Both contractions run on the tensor cores in bf16 with fp32
 * accumulation: dY (if fp32) and Â are rounded to bf16 once (W_q is exact),
 * so each output is within about 2^-7 of Σ|terms| of the exact value.
 * Workspaces (caller-owned) from the matching *_workspace_bytes(). */
size_t bl_ste_grad_input_workspace_bytes(int64_t M, int64_t N, int64_t K);
bl_status bl_ste_grad_input(const void* dY, bl_dtype dy_dtype, int64_t M, int64_t N,
                            const uint8_t* W_packed, const float* gamma, int64_t K,
                            float* dA, void* workspace, size_t ws_bytes, bl_stream_t stream);
size_t bl_ste_grad_weight_workspace_bytes(int64_t M, int64_t N, int64_t K);
bl_status bl_ste_grad_weight(const void* dY, bl_dtype dy_dtype, int64_t M, int64_t N,
                             const int8_t* A_q, const float* gamma_A, int64_t K,
                             const void* W, bl_dtype w_dtype, const float* gamma, float eps,
                             float* dW, void* workspace, size_t ws_bytes, bl_stream_t stream);

/* ---------------------------------------------------------------------------
 * Device error flag. Synchronises `stream`, then returns BL_ERR_TIMEOUT if
 * any kernel of this library on the current device gave up a bounded wait
 * since the last check (and clears the flag), BL_ERR_CUDA if the stream
 * reports an error, else BL_OK.
 */
bl_status bl_check_device_error(bl_stream_t stream);

/* Measurement aid (no counterpart on the pages): launches one empty kernel
 * with exactly the launch shape bl_linear_ex uses for a decode call of
 * (M ≤ bl_gemv_max_tokens(), K, N) — grid, 512 threads, dynamic shared
 * memory, programmatic dependent launch — that only releases its dependents
 * and waits for the previous kernel. A chain of these is the launch-to-launch
 * floor of a dependent decode chain; the GEMV's time above it is its own. */
bl_status bl_probe_pdl_floor(int64_t M, int64_t K, int64_t N, bl_stream_t stream);

/* Self-test of the bounded-wait machinery: launches one tiny kernel that
 * waits on a shared-memory barrier nothing will ever complete, giving up
 * after `limit_ns` nanoseconds (1e3 .. 1e9), which raises the device error
 * flag. Used by the test-suite to exercise the timeout path without hanging
 * or faulting a GPU. */
bl_status bl_selftest_wait_timeout(int64_t limit_ns, bl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
