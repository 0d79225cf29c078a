/*
 * rglru.h — C ABI of the B200 (sm_100a) RG-LRU temporal core library (librglru.so).
 *
 * The layer computed here is the recurrent branch of the Griffin/Hawk recurrent
 * block: a width-4 causal depthwise Conv1D followed by the Real-Gated Linear
 * Recurrent Unit, as defined in "Griffin：将门控线性循环与局部注意力混合以实现高效的
 * 语言模型", §实门线性循环单元 (RG-LRU), Eq. (1)–(4) and the paragraph after them,
 * and §循环块 (recurrent block, Fig. 2(c)):
 *
 *     u_t = conv_b + Σ_{k=0..3} conv_w[k] ⊙ x_{t-3+k}              (Conv1D, width 4)
 *     r_t = σ(W_a u_t + b_a)                                       (1)
 *     i_t = σ(W_x u_t + b_x)                                       (2)
 *     a_t = a^(c r_t),  a = σ(Λ),  c = 8, evaluated in log space    (3)
 *     h_t = a_t ⊙ h_{t-1} + √(1 − a_t²) ⊙ (i_t ⊙ u_t),  y_t = h_t   (4)
 *
 * Around that core the library also offers the recurrent block, its backward, and one
 * Hawk residual layer (RMSNorm, the recurrent block, RMSNorm, gated MLP, residual adds:
 * the same page's §残块 and §MLP块, Fig. 2(a)–(b)), each as a prefill call, with decode
 * steps for the core and for the layer. Every launching call is bracketed by an NVTX
 * range named after it.
 *
 * Conventions shared by every entry point
 *   - R is D_RNN, the channel count. R must be a multiple of 8 (16-byte rows).
 *   - Row-major layouts; "[B][T][R]" means R is contiguous.
 *   - io_dtype selects the type of x, y, u, W_a, W_x and the conv ring:
 *     RGLRU_BF16 (bfloat16) or RGLRU_F32 (float32). Recurrent state h, all gate
 *     arithmetic and accumulation are float32 in both cases. Per-channel parameters
 *     (conv_w, conv_b, b_a, b_x, Λ) are always float32.
 *   - W_a and W_x are dense [R][R] matrices in [out][in] order (z = W u).
 *   - conv_w is [4][R]; tap k multiplies x_{t-3+k} (k = 3 is the current input).
 *   - Every pointer is a DEVICE pointer on the current CUDA device, 16-byte aligned,
 *     unless stated otherwise. The caller owns every buffer, including workspace;
 *     the library never allocates, frees, or synchronises (except
 *     rglru_workspace_status). All work is queued on `stream` (a cudaStream_t;
 *     NULL means the legacy default stream).
 *   - Return value: RGLRU_OK (0) or a negative rglru_status. On an argument error
 *     nothing is launched. Outputs are undefined after any error.
 *   - Not thread-safe for concurrent calls that share a workspace.
 */
#ifndef RGLRU_H_
#define RGLRU_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RGLRU_API __attribute__((visibility("default")))
#else
#define RGLRU_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* rglru_stream_t; /* identical to cudaStream_t */

typedef enum { RGLRU_F32 = 0, RGLRU_BF16 = 1 } rglru_dtype;

typedef enum {
  RGLRU_OK = 0,
  RGLRU_ERR_NULL = -1,      /* a required pointer is NULL */
  RGLRU_ERR_SHAPE = -2,     /* B < 1, T < 1, R < 8, R % 8 != 0, D % 8 != 0, or a size overflows int32 indexing */
  RGLRU_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned */
  RGLRU_ERR_DTYPE = -4,     /* io_dtype not supported by this entry point */
  RGLRU_ERR_WORKSPACE = -5, /* workspace NULL or smaller than the *_workspace_bytes query */
  RGLRU_ERR_CUDA = -6,      /* a CUDA call failed; see rglru_last_cuda_error() */
  RGLRU_ERR_TIMEOUT = -7,   /* a bounded wait inside a kernel gave up (reported by rglru_workspace_status) */
  RGLRU_ERR_DEVICE = -8     /* the current device is not compute capability 10.0 (B200) */
} rglru_status;

/* Per-layer parameters of the Conv1D and the RG-LRU (device pointers). */
typedef struct {
  const float* conv_w; /* [4][R]   Conv1D taps, tap k multiplies x_{t-3+k}           */
  const float* conv_b; /* [R]      Conv1D bias                                         */
  const void* W_a;     /* [R][R]   recurrence-gate weight, io_dtype, Eq. (1)          */
  const float* b_a;    /* [R]      recurrence-gate bias, Eq. (1)                       */
  const void* W_x;     /* [R][R]   input-gate weight, io_dtype, Eq. (2)               */
  const float* b_x;    /* [R]      input-gate bias, Eq. (2)                            */
  const float* Lambda; /* [R]      Λ, with a = σ(Λ), Eq. (3)                           */
} rglru_params;

/* ---------------------------------------------------------------------------------
 * Full-sequence forward (prefill / training forward): Conv1D(4) → RG-LRU over T steps.
 * Eq. (1)–(4) above; the time recurrence is evaluated as a chunked scan (the
 * recurrence is linear in h because neither gate reads h_{t-1}; "Griffin's
 * Compromise: Combining Gated Linear Recurrence with Local Attention", §Hawk,
 * "Parallel scan").
 *
 *   x            [B][T][R] io_dtype, input of the Conv1D
 *   h0           [B][R] float32 initial state, or NULL for zeros
 *   conv_state0  [B][3][R] io_dtype: (x_{-3}, x_{-2}, x_{-1}) in time order, or NULL
 *                for zeros (zero left padding)
 *   y            [B][T][R] io_dtype output, y_t = h_t
 *   h_T          [B][R] float32 final state (may be NULL)
 *   conv_state_T [B][3][R] io_dtype: (x_{T-3}, x_{T-2}, x_{T-1}) in time order (may be NULL)
 *   workspace    device buffer of at least rglru_forward_workspace_bytes(B, T, R, io_dtype)
 *                bytes, 256-byte aligned. It holds u, the gate GEMM's output and the
 *                scan's chunk carries; its contents need no initialisation.
 * Kernels, RGLRU_BF16: conv (x → u, bf16), the 2-SM tcgen05 gate GEMM whose epilogue
 * applies the gates and the log-space decay and writes the recurrence coefficients
 * d = 1 − a_t (fp16) and b_t = √(1 − a_t²)·i_t·u_t (bf16) (rglru_gate_coeffs), then the
 * chunked scan of h_t = (1 − d)·h_{t−1} + b_t (rglru_scan_coeffs). RGLRU_F32: conv, the
 * FFMA gate GEMM writing the packed pre-activations (rglru_gate_proj), then the scan that
 * recomputes u and applies the gates and the decay itself (rglru_scan).
 * Domain: every finite input whose Conv1D output u, pre-activations and states are finite
 * in float32 gives finite outputs (no format narrower than the IO type holds u-scaled
 * values). With bf16 IO the gates are evaluated from the bf16-rounded u: where W u is so
 * large that a pre-activation's rounding error crosses σ's transition, r and i differ from
 * the unrounded ones (a property of the bf16 operand, not of the scan).
 * --------------------------------------------------------------------------------- */
RGLRU_API size_t rglru_forward_workspace_bytes(int B, int T, int R, int io_dtype);
/* How many kernels rglru_forward launches for this shape (0 for invalid arguments): 2 when
 * it takes the gate GEMM with the scan fused into its epilogue (bf16 IO, T a multiple of 128,
 * R ≥ 4096, where that epilogue hides behind the tile's MMAs; see rglru_gate_scan), else 3
 * (Conv1D, the gate GEMM forming the coefficients, the scan). */
RGLRU_API int rglru_forward_kernels(int B, int T, int R, int io_dtype);
RGLRU_API int rglru_forward(const rglru_params* params, const void* x, const float* h0, const void* conv_state0,
                  void* y, float* h_T, void* conv_state_T, int B, int T, int R, int io_dtype,
                  void* workspace, size_t workspace_bytes, rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * One decode step on a carried state ("Griffin's Compromise…", §Hawk: generation reads
 * and writes only the current token and a fixed-size state), Eq. (1)–(4) at one t.
 *
 *   x_t         [B][R] io_dtype current input
 *   conv_state  [B][3][R] io_dtype ring of the last three inputs, updated IN PLACE:
 *               slot (step mod 3) holds x_{t-3}, slot (step+1) mod 3 holds x_{t-2},
 *               slot (step+2) mod 3 holds x_{t-1}; on return slot (step mod 3) holds x_t.
 *               A state in time order (as rglru_forward writes it) is the ring at any
 *               step ≡ 0 (mod 3).
 *   step        ≥ 0, the ring position described above
 *   h           [B][R] float32 state, updated IN PLACE (h_{t-1} → h_t)
 *   y_t         [B][R] io_dtype output (= new h)
 *   workspace   at least rglru_step_workspace_bytes(B, R, io_dtype) bytes (holds u_t, in
 *               bf16 for the gate GEMM and in float32 for the state update)
 * io_dtype must be RGLRU_BF16 (the tensor-core path) for this entry point.
 * --------------------------------------------------------------------------------- */
RGLRU_API size_t rglru_step_workspace_bytes(int B, int R, int io_dtype);
RGLRU_API int rglru_step(const rglru_params* params, const void* x_t, void* conv_state, float* h, void* y_t, int B,
               int R, int64_t step, int io_dtype, void* workspace, size_t workspace_bytes,
               rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Recurrent block ("Griffin：…", §循环块, Fig. 2(c)):
 *   v = x W_1ᵀ, g = x W_2ᵀ                (two D → D_RNN linears, no bias)
 *   h = RG-LRU(Conv1D(v))                  (as rglru_forward, zero conv history)
 *   out = (h ⊙ GeLU(g)) W_oᵀ               (exact erf GeLU; D_RNN → D linear, no bias)
 *
 *   x [B][T][D], W_1 and W_2 [R][D], W_o [D][R], out [B][T][D]: all bfloat16.
 *   h0 [B][R] float32 or NULL; h_T [B][R] float32 or NULL.
 *   io_dtype must be RGLRU_BF16. D % 8 == 0.
 * --------------------------------------------------------------------------------- */
RGLRU_API size_t rglru_block_workspace_bytes(int B, int T, int D, int R, int io_dtype);
RGLRU_API int rglru_block_forward(const rglru_params* params, const void* W_1, const void* W_2, const void* W_o,
                        const void* x, const float* h0, void* out, float* h_T, int B, int T, int D, int R,
                        int io_dtype, void* workspace, size_t workspace_bytes, rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Hawk residual layer ("Griffin：…", §残块, Fig. 2(a); §MLP块, Fig. 2(b)): the recurrent
 * block as the temporal-mixing block, each component pre-normed by RMSNorm (Zhang &
 * Sennrich) and merged with the skip connection from its own RMSNorm input:
 *   y   = x + RecurrentBlock(RMSNorm₁(x))          (the recurrent block above)
 *   out = y + (GeLU(n W_gateᵀ) ⊙ n W_upᵀ) W_downᵀ,  n = RMSNorm₂(y)
 *   RMSNorm(v) = v / √(mean_j v_j² + eps) ⊙ scale    (per row of D channels)
 *
 *   x, out      [B][T][D] bfloat16, distinct buffers
 *   W_1, W_2    [R][D]; W_o [D][R]; W_gate, W_up [H][D]; W_down [D][H]: bfloat16,
 *               row-major [out][in], no biases (H = M·D; the pages use M = 3)
 *   norm1_scale, norm2_scale  [D] float32 gains
 *   h0, h_T     [B][R] float32 or NULL, as in rglru_block_forward
 *   eps         RMSNorm ε, 0 ≤ eps ≤ 1 (1e-6 in the tests)
 *   workspace   at least rglru_layer_workspace_bytes(B, T, D, R, H, io_dtype) bytes,
 *               256-byte aligned (the block's buffers plus four [B·T][D] and two
 *               [B·T][H] bf16 activations)
 * The residual stream y is rounded to bf16 once, as it is stored; every norm, GeLU and
 * accumulation is float32. io_dtype must be RGLRU_BF16; D, R, H multiples of 8.
 * Errors as everywhere: RGLRU_ERR_SHAPE also for out == x or eps outside [0, 1].
 * --------------------------------------------------------------------------------- */
typedef struct rglru_layer_weights {
  const float* norm1_scale; /* [D] RMSNorm gain ahead of the recurrent block */
  const void* W_1;          /* [R][D] */
  const void* W_2;          /* [R][D] */
  const void* W_o;          /* [D][R] */
  const float* norm2_scale; /* [D] RMSNorm gain ahead of the MLP */
  const void* W_gate;       /* [H][D], the GeLU branch */
  const void* W_up;         /* [H][D] */
  const void* W_down;       /* [D][H] */
} rglru_layer_weights;
RGLRU_API size_t rglru_layer_workspace_bytes(int B, int T, int D, int R, int H, int io_dtype);
RGLRU_API int rglru_layer_forward(const rglru_params* params, const rglru_layer_weights* weights, const void* x,
                                  const float* h0, void* out, float* h_T, int B, int T, int D, int R, int H,
                                  float eps, int io_dtype, void* workspace, size_t workspace_bytes,
                                  rglru_stream_t stream);
/* One decode step of the same layer on a carried state (the decode form of the
 * recurrent block: "Griffin's Compromise…", §Hawk — generation reads and writes only the
 * current token and a fixed-size state):
 *   y   = x_t + ((RG-LRU step of Conv1D(v)) ⊙ GeLU(g)) W_oᵀ,  v = n W_1ᵀ, g = n W_2ᵀ, n = RMSNorm₁(x_t)
 *   out_t = y + MLP(RMSNorm₂(y))
 *   x_t, out_t  [B][D] bfloat16, distinct
 *   conv_state  [B][3][R] bfloat16 ring of the last three inputs of the Conv1D (the v
 *               branch), updated IN PLACE exactly as rglru_step updates its ring
 *   h           [B][R] float32 RG-LRU state, updated IN PLACE
 *   step        ≥ 0, the ring position (as rglru_step)
 *   weights, eps, D, R, H as rglru_layer_forward
 *   workspace   at least rglru_layer_step_workspace_bytes(B, D, R, H, io_dtype) bytes,
 *               256-byte aligned
 * io_dtype must be RGLRU_BF16. Errors as rglru_layer_forward, plus RGLRU_ERR_SHAPE for
 * step < 0. */
RGLRU_API size_t rglru_layer_step_workspace_bytes(int B, int D, int R, int H, int io_dtype);
RGLRU_API int rglru_layer_step(const rglru_params* params, const rglru_layer_weights* weights, const void* x_t,
                               void* conv_state, float* h, void* out_t, int B, int D, int R, int H, int64_t step,
                               float eps, int io_dtype, void* workspace, size_t workspace_bytes,
                               rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Griffin's local multi-query attention, one decode step ("Griffin：…", §时间混合块:
 * MQA with H query heads of D_head = 128, H·D_head = D, one key/value head shared by all
 * of them, RoPE as the relative position embedding, sliding-window attention whose KV
 * cache is bounded by the window; "Griffin's Compromise…", §"Griffin: Attention for Recent
 * Memory, Recurrence for Long-Range Flow": window 1024, one
 * local-attention residual block after every two recurrent ones). At position `pos`:
 *   q = x_t W_qᵀ, k = x_t W_kᵀ, v = x_t W_vᵀ;  q, k rotated by RoPE at `pos`
 *   (pair i = (x_{2i}, x_{2i+1}) turned by pos·θ_i, θ_i = 10000^(−2i/128));
 *   (k, v) stored into ring slot (pos mod window);
 *   o_h = Σ_s softmax_s(q_h·k_s / √128) v_s over the window's positions
 *         max(0, pos − window + 1) … pos;  out_t = o W_oᵀ.
 *
 *   weights.W_qkv  [(H+2)·128][D] bf16, row-major [out][in]: the H·128 rows of W_q (head h
 *                  in rows 128h … 128h+127), then the 128 rows of W_k, then of W_v
 *   weights.W_o    [D][H·128] bf16
 *   x_t, out_t     [B][D] bf16
 *   k_ring         [B][window][128] bf16, rotated keys, slot-major; updated IN PLACE
 *   v_ring         [B][window][128] bf16, values, slot-major; updated IN PLACE. Slots
 *                  holding no position yet (pos < window − 1) are never read, so the rings
 *                  need no initialisation.
 *   pos            ≥ 0, the position of x_t; the rings hold positions pos − window … pos − 1
 *   workspace      at least rglru_attention_step_workspace_bytes(B, D, window) bytes,
 *                  256-byte aligned
 * D a multiple of 128 with D/128 ≤ 64; window a multiple of 128 (≤ 65536); B ≤ 65535.
 * Errors as everywhere (RGLRU_ERR_SHAPE for any other D, window, B or pos < 0); a timeout
 * of a bounded wait is reported by rglru_workspace_status(workspace, stream).
 * --------------------------------------------------------------------------------- */
typedef struct {
  const void* W_qkv; /* [(H+2)·128][D] */
  const void* W_o;   /* [D][H·128]     */
} rglru_attention_weights;
RGLRU_API size_t rglru_attention_step_workspace_bytes(int B, int D, int window);
RGLRU_API int rglru_attention_step(const rglru_attention_weights* weights, const void* x_t, void* k_ring,
                                   void* v_ring, void* out_t, int B, int D, int window, int64_t pos,
                                   void* workspace, size_t workspace_bytes, rglru_stream_t stream);
/* The residual block of Griffin with local attention as its temporal-mixing block, one
 * decode step (§残块, Fig. 2(a), as the Hawk layer above with local MQA in place of the
 * recurrent block):
 *   y = x_t + LocalMQA(RMSNorm₁(x_t)),   out_t = y + (GeLU(n W_gateᵀ) ⊙ n W_upᵀ) W_downᵀ,
 *   n = RMSNorm₂(y)
 * x_t, out_t [B][D] bf16, distinct; k_ring, v_ring, pos, window as rglru_attention_step;
 * W_gate, W_up [H][D], W_down [D][H] bf16 (H = M·D, the MLP width); eps as the Hawk layer.
 * workspace: at least rglru_attention_layer_step_workspace_bytes(B, D, H, window) bytes. */
typedef struct {
  const float* norm1_scale; /* [D] */
  const void* W_qkv;        /* [(D/128 + 2)·128][D] */
  const void* W_o;          /* [D][D] */
  const float* norm2_scale; /* [D] */
  const void* W_gate;       /* [H][D] */
  const void* W_up;         /* [H][D] */
  const void* W_down;       /* [D][H] */
} rglru_attention_layer_weights;
RGLRU_API size_t rglru_attention_layer_step_workspace_bytes(int B, int D, int H, int window);
RGLRU_API int rglru_attention_layer_step(const rglru_attention_layer_weights* weights, const void* x_t,
                                         void* k_ring, void* v_ring, void* out_t, int B, int D, int H, int window,
                                         int64_t pos, float eps, void* workspace, size_t workspace_bytes,
                                         rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Backward of rglru_forward for bf16 IO: the gradients of a scalar loss ℓ with respect to
 * the input, the parameters, the initial state and the conv history, given ∂ℓ/∂y and
 * ∂ℓ/∂h_T. Reverse-mode differentiation of Eq. (1)–(4) above (with the log-space decay
 * of the paragraph after them: log a_t = r_t·c·log σ(Λ)) and of the Conv1D of §循环块:
 * with g_t = ∂ℓ/∂h_t = dy_t + a_{t+1} g_{t+1} (g after the last step = dh_T),
 *   ∂z_a = (g h_{t-1} a_t r_t − g i_t u_t a_t² r_t/√(1−a_t²))·c·log σ(Λ)·(1 − r_t),
 *   ∂z_x = g √(1−a_t²) u_t · i_t (1 − i_t),  ∂u_t = g √(1−a_t²) i_t + ∂z_a W_a + ∂z_x W_x,
 *   ∂W_a = Σ_t ∂z_aᵀ u_t, ∂b_a = Σ_t ∂z_a (same for x), ∂Λ = Σ (∂log a_t) c r_t · σ(−Λ),
 *   ∂h0 = a_0 g_0, and the Conv1D's transpose for ∂x, the taps, the bias and the history.
 * u and the gate pre-activations are recomputed from x (or, in rglru_backward_saved, the
 * pre-activations come from rglru_forward_train); h_{t-1} is read from y.
 *   params        as rglru_forward (W_a, W_x bf16)
 *   x             [B][T][R] bf16, the forward's input
 *   y             [B][T][R] bf16, the forward's output for the same x, h0, conv_state0
 *   dy            [B][T][R] bf16, ∂ℓ/∂y
 *   h0            [B][R] float32 or NULL (zeros), as in the forward
 *   dh_T          [B][R] float32 or NULL (zeros), ∂ℓ/∂h_T
 *   conv_state0   [B][3][R] bf16 or NULL (zeros), as in the forward
 *   grads         output buffers (all 16-byte aligned; the library writes every one, and
 *                 zeroes the accumulated ones first): dx [B][T][R] bf16; dconv_state0
 *                 [B][3][R] bf16 or NULL; dconv_w [4][R], dconv_b, db_a, db_x, dLambda [R],
 *                 dW_a, dW_x [R][R] (row-major [out][in]) and dh0 [B][R] (or NULL) float32
 *   workspace     at least rglru_backward_workspace_bytes(B, T, R) bytes, 256-byte aligned
 * Shapes: as rglru_forward, and B·⌈T/64⌉ ≤ 65535 (RGLRU_ERR_SHAPE).
 * The accumulated outputs (the taps, biases and Λ) are summed with atomics, so their
 * last bits may vary between runs; everything else is deterministic.
 * --------------------------------------------------------------------------------- */
typedef struct {
  void* dx;           /* [B][T][R] bf16                          */
  void* dconv_state0; /* [B][3][R] bf16, or NULL                 */
  float* dconv_w;     /* [4][R]                                  */
  float* dconv_b;     /* [R]                                     */
  float* dW_a;        /* [R][R]                                  */
  float* db_a;        /* [R]                                     */
  float* dW_x;        /* [R][R]                                  */
  float* db_x;        /* [R]                                     */
  float* dLambda;     /* [R]                                     */
  float* dh0;         /* [B][R], or NULL                         */
} rglru_grads;
RGLRU_API size_t rglru_backward_workspace_bytes(int B, int T, int R);
RGLRU_API int rglru_backward(const rglru_params* params, const void* x, const void* y, const void* dy,
                             const float* h0, const float* dh_T, const void* conv_state0, const rglru_grads* grads,
                             int B, int T, int R, void* workspace, size_t workspace_bytes, rglru_stream_t stream);

/* Training pair: rglru_forward_train is rglru_forward for bf16 IO that also writes the gate
 * pre-activations z = u W_aᵀ + b_a, u W_xᵀ + b_x (bf16, in an internal packed layout) into
 * `saved`, at least rglru_saved_bytes(B, T, R) bytes, 16-byte aligned (0 for invalid
 * shapes). rglru_backward_saved is rglru_backward reading them from `saved` instead of
 * recomputing them with the gate GEMM: the same inputs and outputs, bit for bit the same
 * results (the saved values are those the recomputation forms). The pages keep the
 * backward's inputs open; this pair trades rglru_saved_bytes of memory between the two calls
 * for one of the backward's three gate-sized GEMMs. Errors as rglru_forward and
 * rglru_backward, plus RGLRU_ERR_NULL for a null `saved`. */
RGLRU_API size_t rglru_saved_bytes(int B, int T, int R);
RGLRU_API int rglru_forward_train(const rglru_params* params, const void* x, const float* h0, const void* conv_state0,
                                  void* y, float* h_T, void* conv_state_T, void* saved, int B, int T, int R,
                                  void* workspace, size_t workspace_bytes, rglru_stream_t stream);
RGLRU_API int rglru_backward_saved(const rglru_params* params, const void* x, const void* y, const void* dy,
                                   const float* h0, const float* dh_T, const void* conv_state0, const void* saved,
                                   const rglru_grads* grads, int B, int T, int R, void* workspace,
                                   size_t workspace_bytes, rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * The stages of rglru_forward, callable one by one (for per-kernel timing and for
 * testing each stage against the oracle). rglru_forward runs exactly rglru_conv1d, then
 * for RGLRU_BF16 rglru_gate_coeffs and rglru_scan_coeffs, for RGLRU_F32 rglru_gate_proj
 * and rglru_scan.
 *
 * rglru_conv1d: u = Conv1D(x) (§循环块). x, u [B][T][R] io_dtype; conv_state0 as in
 *   rglru_forward (NULL = zeros); conv_state_T may be NULL.
 *
 * rglru_gate_proj: z = u [W_a | W_x]ᵀ + [b_a | b_x] for N_tok = B·T rows (Eq. (1)–(2)
 *   arguments of σ). z is written in the PACKED gate layout: row n has
 *   rglru_gate_pitch(R) elements; channel c's recurrence-gate pre-activation sits at
 *   column 256·(c / 128) + (c % 128) and its input-gate pre-activation at
 *   256·(c / 128) + 128 + (c % 128). Columns of a partial last block are unused.
 *   z has io_dtype (bf16 rounding of the fp32 accumulator for RGLRU_BF16).
 *
 * rglru_scan: Eq. (1)–(4) given x and the packed z: recomputes u from x (fp32),
 *   applies σ, the log-space decay and the chunked recurrence. If gate_g is non-NULL
 *   ([B][T][R] io_dtype) the output is y_t = h_t ⊙ GeLU(g_t) (the block's product),
 *   otherwise y_t = h_t. h_T [B][R] (may be NULL) is the final state in both cases.
 *   workspace: at least rglru_scan_workspace_bytes(B, T, R, io_dtype) bytes.
 * --------------------------------------------------------------------------------- */
RGLRU_API int rglru_conv1d(const float* conv_w, const float* conv_b, const void* x, const void* conv_state0, void* u,
                 void* conv_state_T, int B, int T, int R, int io_dtype, rglru_stream_t stream);
RGLRU_API int64_t rglru_gate_pitch(int R);
RGLRU_API int rglru_gate_proj(const void* u, const void* W_a, const float* b_a, const void* W_x, const float* b_x,
                    void* z, int64_t N_tok, int R, int io_dtype, rglru_stream_t stream);
RGLRU_API size_t rglru_scan_workspace_bytes(int B, int T, int R, int io_dtype);
RGLRU_API int rglru_scan(const rglru_params* params, const void* x, const void* z, const void* conv_state0,
               const float* h0, const void* gate_g, void* y, float* h_T, int B, int T, int R, int io_dtype,
               void* workspace, size_t workspace_bytes, rglru_stream_t stream);

/* rglru_gate_coeffs (bf16 u and weights): the gate GEMM with the gates applied in its
 *   epilogue ("Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §实门线性循环单元,
 *   Eq. (1)–(4)): with z as in rglru_gate_proj, r = σ(z_a), i = σ(z_x),
 *   log a_t = r·c·log σ(Λ), it writes the recurrence coefficients d = 1 − a_t and
 *   b_t = √(1 − a_t²)·i·u_t (so that h_t = (1 − d)·h_{t−1} + b_t) in the packed layout of
 *   z: d as IEEE fp16 in the recurrence-gate places, b_t as bf16 in the input-gate places.
 *   u is the bf16 Conv1D output [N_tok][R] (the GEMM's operand; the same u enters b_t).
 *   g is [N_tok][rglru_gate_pitch(R)] 16-bit words, 16-byte aligned. d ∈ [0, 1] keeps
 *   fp16's 11 significant bits (its relative error multiplies into every carried state);
 *   b_t, which scales with u_t, keeps bf16's exponent range, so every finite bf16 u gives
 *   a finite b_t (|b_t| ≤ |u_t|, since √(1 − a_t²)·i ≤ 1).
 *
 * rglru_scan_coeffs: the chunked recurrence h_t = (1 − d)·h_{t−1} + b_t over those
 *   coefficients, for bf16 IO: y_t = h_t, or h_t ⊙ GeLU(gate_g_t) when gate_g is non-NULL,
 *   and h_T, exactly as rglru_scan. It reads neither x nor the parameters. g [B·T rows] as
 *   written by rglru_gate_coeffs; h0, gate_g, y, h_T and the workspace as rglru_scan with
 *   io_dtype = RGLRU_BF16.
 */
RGLRU_API int rglru_gate_coeffs(const rglru_params* params, const void* u, void* g, int64_t N_tok, int R,
                                rglru_stream_t stream);
RGLRU_API int rglru_scan_coeffs(const void* g, const float* h0, const void* gate_g, void* y, float* h_T, int B, int T,
                                int R, void* workspace, size_t workspace_bytes, rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * rglru_scan without a workspace, for callers that cannot allocate device memory: a
 * custom operator whose host framework hands it only its input and output buffers, a
 * serving process whose memory is fully reserved at start-up, or a latency-critical loop
 * that must not call cudaMalloc (which can synchronise the device). The paper has no
 * counterpart to this entry point; it exists for those callers only.
 *
 * Same arguments, checks and results as rglru_scan, minus the workspace. The scan's
 * scratch (status word, tile ticket, published chunk states and chunk maps) is a fixed
 * 8 MiB array in the library's device memory, which every GPU that loads librglru.so holds
 * until the process exits. A problem fits if
 *   256 + ⌈n_tiles·4·CW / 256⌉·256 + n_tiles·8·CW ≤ 8 MiB,
 * with n_tiles = B·⌈R/CW⌉·⌈T/64⌉ and CW = 128 channels for bf16, 64 for float32: at most
 * 5461 bf16 tiles (e.g. B=1, T=10880, R=4096) or 10922 float32 tiles. Larger problems are
 * rejected with RGLRU_ERR_WORKSPACE before anything is launched. Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library call.
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream capture.
 * All calls on a device share the one array, and it keeps the last call's contents (each
 * call clears the parts that must start at zero, its status word included): calls that
 * overlap on the GPU — on different streams, or from different threads — race and give
 * wrong results. A timeout of the call's bounded waits is reported by
 * rglru_scan_noalloc_status, which synchronises `stream`, reads the array's status word
 * and clears it (RGLRU_OK or RGLRU_ERR_TIMEOUT); the next call clears it too.
 * --------------------------------------------------------------------------------- */
RGLRU_API int rglru_scan_noalloc(const rglru_params* params, const void* x, const void* z, const void* conv_state0,
                                 const float* h0, const void* gate_g, void* y, float* h_T, int B, int T, int R,
                                 int io_dtype, rglru_stream_t stream);
RGLRU_API int rglru_scan_noalloc_status(rglru_stream_t stream);

/* The gate GEMM with the RG-LRU scan fused into its epilogue (Eq. (1)–(4)): y and h_T
 * from u = Conv1D(x) in bf16 [B][T][R] (the tensor-core operand, also the u of
 * b_t = √(1−a_t²)·i_t·u_t). The recurrence coefficients stay in registers in float32 (no
 * fp16/bf16 storage rounding of d and b_t, unlike the three-kernel path). bf16 only; T
 * must be a multiple of 128 (each 128-step chunk of a batch row is one accumulator tile).
 * h0 and h_T as in rglru_forward. workspace: at least
 * rglru_gate_scan_workspace_bytes(B, T, R, io_dtype) bytes, 256-byte aligned (chunk carries;
 * zeroed by the call). */
RGLRU_API size_t rglru_gate_scan_workspace_bytes(int B, int T, int R, int io_dtype);
RGLRU_API int rglru_gate_scan(const rglru_params* params, const void* u, const float* h0, void* y, float* h_T, int B,
                              int T, int R, int io_dtype, void* workspace, size_t workspace_bytes,
                              rglru_stream_t stream);

/* Dense bf16 GEMM C[M][N] = A[M][K] · B[N][K]ᵀ on the tcgen05 tensor cores (fp32
 * accumulate, bf16 store), the kernel behind the block's linears. K % 8 == 0, N % 8 == 0. */
RGLRU_API int rglru_gemm_bf16(const void* A, const void* Bm, void* C, int64_t M, int N, int K, rglru_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Status and diagnostics
 * --------------------------------------------------------------------------------- */
/* Synchronises `stream`, reads and clears the device status word that kernels using
 * `workspace` (forward, scan, block) write; returns RGLRU_OK or RGLRU_ERR_TIMEOUT. */
RGLRU_API int rglru_workspace_status(void* workspace, rglru_stream_t stream);
/* Text for a status code (static storage). */
RGLRU_API const char* rglru_strerror(int status);
/* The cudaError_t of the last RGLRU_ERR_CUDA on this thread (0 if none). */
RGLRU_API int rglru_last_cuda_error(void);
/* TESTING ONLY. Makes every later scan (rglru_scan, rglru_forward, rglru_block_forward)
 * leave the chunk carry of tile `tile` unpublished, so that the CTAs waiting for it run
 * into their bounded wait (about one second), give up, and set RGLRU_ERR_TIMEOUT in the
 * workspace status word; the outputs are then wrong but every kernel ends. Tile index =
 * ((b · n_channel_blocks + channel_block) · n_time_chunks + time_chunk) with 64-step
 * time chunks and 128 (bf16) or 64 (f32) channels per block. A negative value turns the
 * injection off. Always returns RGLRU_OK. */
RGLRU_API int rglru_debug_scan_stall(int64_t tile);
/* Library version: major*10000 + minor*100 + patch. */
RGLRU_API int rglru_version(void);

#ifdef __cplusplus
}
#endif
#endif /* RGLRU_H_ */
