/*
 * oracle.h -- plain single-threaded CPU oracle for the ternary routed-expert
 * MoE hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this code; only the test suite, the package smoke check and the
 * benchmark's timed CPU-baseline leg use it.  It shares no source, header,
 * table or constant with the CUDA library under bit_moe_b200/.
 *
 * What it computes, and where each piece comes from:
 *   - routed-expert weights are ternary values (Parallax 8B kappa article,
 *     section "Что именно доступно") kept compressed in blocks and multiplied
 *     against int8-quantized activations (Parakon Runtime README, section
 *     "How it works"); the block format itself is not printed on any page, so
 *     it is fixed here as: 256 weights per block, absmean scale rounded to
 *     fp16, five base-3 digits per byte (52 bytes per block);
 *   - int8 activations carry one fp32 scale per 32 values (pxq_llama README,
 *     section "PXQ vs MXFP4": one scale fixup per 32-value block);
 *   - all top-k experts of a token are evaluated, none dropped
 *     (llama-modchip page, "Key highlights");
 *   - the expert FFN is gate/up with a SiLU unary, then down (pxq_llama README,
 *     "Updates -- 2026-07-28", the up_gate_unary item);
 *   - two more routed-weight formats of the pxq_llama README ("What's PXQ?"):
 *     1-bit sign codes, and two-level (E16) scales on the ternary digits;
 *   - a shared expert kept at higher precision beside the routed ones
 *     (llama-modchip page, "The interesting bit"), in 8-bit blocks.
 * Every other detail is a reading of those passages; each function below says
 * which.
 *
 * Floating point: sums that define a result are taken in fp64; where a float
 * decides an integer (a scale rounded to fp16, an int8 code, a top-k order)
 * the decision is taken in the precision stated at that function, which is
 * the precision the method fixes.  Built with -ffp-contract=off.
 */
#ifndef BITMOE_ORACLE_H
#define BITMOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Format constants (see orc_quantize_weights). */
#define ORC_BLOCK 256       /* weights per ternary block                 */
#define ORC_BLOCK_WORDS 13  /* 32-bit words of packed digits per block   */
#define ORC_PANEL 32        /* rows interleaved word by word in storage  */
#define ORC_QBLOCK 32       /* activations per int8 block                */

/* ---- IEEE binary16 ---------------------------------------------------- */
/* Round a double to the nearest binary16, ties to even; overflow gives inf. */
uint16_t orc_f16_from_f64(double x);
/* Exact widening of a binary16 bit pattern to float. */
float orc_f16_to_f32(uint16_t h);

/* ---- base-3 byte -------------------------------------------------------- */
/* Five digits t[0..4] in {0,1,2}, t[0] most significant: v = sum t_i 3^(4-i),
 * stored as the fixed-point fraction u = ceil(v * 256 / 243).              */
uint8_t orc_trit_byte_encode(const int t[5]);
/* Inverse of the above by plain integer arithmetic: v = floor(u*243/256),
 * then repeated division by 3.  Returns -1 if u encodes no valid v.        */
int orc_trit_byte_decode(uint8_t u, int t[5]);

/* ---- weight storage ----------------------------------------------------- */
int64_t orc_trit_words(int64_t rows, int64_t k);   /* rows*(k/256)*13 */
int64_t orc_scale_count(int64_t rows, int64_t k);  /* rows*(k/256)    */
/* Index of packed word w (0..12) of block b of row r. */
int64_t orc_word_index(int64_t k, int64_t r, int64_t b, int w);
/* Index of the fp16 scale of block b of row r. */
int64_t orc_scale_index(int64_t k, int64_t r, int64_t b);

/* Quantize w [rows][k] (row-major fp32) to ternary blocks.  Returns 0, or -1
 * when rows % 32 or k % 256 is nonzero.                                    */
int orc_quantize_weights(const float* w, int64_t rows, int64_t k,
                         uint32_t* trits, uint16_t* scales);
/* Expand rows [row0, row0+nrows) to q [nrows][k] in {-1,0,1} and the fp32
 * value of each block scale s [nrows][k/256].  Returns 0, or -1 on a bad
 * shape or an undecodable byte.                                            */
int orc_unpack_weights(const uint32_t* trits, const uint16_t* scales,
                       int64_t rows, int64_t k, int64_t row0, int64_t nrows,
                       int8_t* q, float* s);

/* ---- 1-bit sign codes -------------------------------------------------- */
/* The 1-bit tier of the pxq_llama README ("What's PXQ?", the PXQ1 row: sign
 * codes times scales).  Reading: the same 256-weight blocks, 32-row panels
 * and fp16 absmean scale as the ternary format; q = -1 where w < 0, else +1;
 * one bit per weight in ORC_SIGN_WORDS 32-bit words per block: word j holds
 * weights 32j .. 32j+31, weight 32j + 4i + l in bit 8l + i, a set bit
 * meaning +1.  34 bytes per block (1.0625 bits per weight).                */
#define ORC_SIGN_WORDS 8
int64_t orc_sign_words(int64_t rows, int64_t k);   /* rows*(k/256)*8 */
/* Index of code word w (0..7) of block b of row r. */
int64_t orc_sign_word_index(int64_t k, int64_t r, int64_t b, int w);
/* Quantize w [rows][k] to sign codes; scales as orc_quantize_weights.
 * Returns 0, or -1 when rows % 32 or k % 256 is nonzero.                  */
int orc_quantize_weights_sign(const float* w, int64_t rows, int64_t k,
                              uint32_t* codes, uint16_t* scales);
/* Expand rows [row0, row0+nrows) to q [nrows][k] in {-1,+1} and the block
 * scales s [nrows][k/256].  Returns 0, or -1 on a bad shape.              */
int orc_unpack_weights_sign(const uint32_t* codes, const uint16_t* scales,
                            int64_t rows, int64_t k, int64_t row0,
                            int64_t nrows, int8_t* q, float* s);

/* ---- two-level scales (E16) ------------------------------------------------ */
/* The E16-row scales of the pxq_llama README ("What's PXQ?": a per-row fp16
 * anchor plus a 4-bit sub-scale per 16-element block), read onto the
 * ternary digits: per row A = fp16_RNE(max over its 16-weight blocks of
 * mean|w|, fp64); per 16-weight block h a code c_h in 0..15 with scale
 * s_h = A * (c_h + 1) / 16, c_h = clamp(rint(16 * m_h / A) - 1, 0, 15)
 * (m_h the block's mean|w| in fp64, A as a double; c_h = 0 when A = 0);
 * q = sign(w) where |w| >= s_h / 2 in fp32, else 0.  Storage: the base-3
 * words of the ternary format (orc_word_index), ORC_E16_WORDS words of
 * codes per 256 weights (word u of block b holds 16-blocks 8u..8u+7, block
 * 8u + v in bits 4v..4v+3; interleaved over 32-row panels like the digits)
 * and one fp16 anchor per row.                                            */
#define ORC_E16_WORDS 2
int64_t orc_e16_code_words(int64_t rows, int64_t k);  /* rows*(k/256)*2 */
/* Index of code word u (0..1) of block b of row r. */
int64_t orc_e16_code_index(int64_t k, int64_t r, int64_t b, int u);
/* Quantize w [rows][k]: trits [orc_trit_words], codes [orc_e16_code_words],
 * anchors [rows].  Returns 0, or -1 when rows % 32 or k % 256 is nonzero. */
int orc_quantize_weights_e16(const float* w, int64_t rows, int64_t k,
                             uint32_t* trits, uint32_t* codes,
                             uint16_t* anchors);
/* Expand rows [row0, row0+nrows) to q [nrows][k] in {-1,0,1} and the fp32
 * scale of every 16-weight block s16 [nrows][k/16] (A * (c+1) / 16, exact
 * in fp32).  Returns 0, or -1 on a bad shape or an undecodable byte.     */
int orc_unpack_weights_e16(const uint32_t* trits, const uint32_t* codes,
                           const uint16_t* anchors, int64_t rows, int64_t k,
                           int64_t row0, int64_t nrows, int8_t* q,
                           float* s16);
/* out[r] = sum_j xd[j] * sum_{16-blocks h in activation block j}
 *          s16[r][h] * sum_{k in h} q[r][k] * xq[k], in fp64.             */
void orc_matvec_e16(const int8_t* q, const float* s16, int64_t rows,
                    int64_t k, const int8_t* xq, const float* xd,
                    double* out);

/* ---- activations ---------------------------------------------------------- */
/* x [ntok][k] -> xq [ntok][k] int8, xd [ntok][k/32] fp32.  Returns -1 if
 * k % 32 != 0.                                                             */
int orc_quant_act_q8(const float* x, int64_t ntok, int64_t k, int8_t* xq,
                     float* xd);

/* ---- block sums and mat-vec ----------------------------------------------- */
/* isum [rows][k/32] = per-32-block int32 dot products of q rows with xq.   */
void orc_blocksums(const int8_t* q, int64_t rows, int64_t k, const int8_t* xq,
                   int32_t* isum);
/* out[r] = sum_b s[r][b] * sum_{j in b} xd[j] * isum[r][j], in fp64.       */
void orc_matvec(const int8_t* q, const float* s, int64_t rows, int64_t k,
                const int8_t* xq, const float* xd, double* out);

/* ---- router ------------------------------------------------------------------ */
/* logits [ntok][E] in fp32, in the fixed evaluation order described at the
 * definition.  Returns -1 if hidden % 32 != 0.                             */
int orc_router_logits(const float* x, const float* wr, int64_t ntok,
                      int64_t hidden, int64_t n_experts, float* logits);
/* top-k experts by logit (descending, ties to the lower id) and their
 * softmax weights renormalised over the k selected, in fp64.              */
int orc_route_topk(const float* x, const float* wr, int64_t ntok,
                   int64_t hidden, int64_t n_experts, int64_t top_k,
                   int32_t* idx, double* wts);

/* ---- expert FFN ------------------------------------------------------------- */
typedef struct {
  int64_t hidden, ffn, n_experts, top_k;
  const uint32_t* gate_trits; const uint16_t* gate_scales; /* rows E*ffn, k hidden */
  const uint32_t* up_trits;   const uint16_t* up_scales;   /* rows E*ffn, k hidden */
  const uint32_t* down_trits; const uint16_t* down_scales; /* rows E*hidden, k ffn */
  int64_t format; /* ORC_FORMAT_TERNARY, ORC_FORMAT_SIGN (the *_trits
                     pointers then hold sign code words) or ORC_FORMAT_E16
                     (the *_scales pointers then hold the per-row anchors)  */
  const uint32_t* gate_codes; /* ORC_FORMAT_E16: the 4-bit sub-scale words */
  const uint32_t* up_codes;
  const uint32_t* down_codes;
} orc_layer;
#define ORC_FORMAT_TERNARY 0
#define ORC_FORMAT_SIGN 1
#define ORC_FORMAT_E16 2

/* y [ntok][hidden] (fp64) = sum over slots j (in slot order) of
 * wts[t][j] * FFN_{idx[t][j]}(x_t).  Optional (may be NULL) debug outputs,
 * each [ntok][top_k][...]: g and u (fp64, [ffn]), aq (int8, [ffn]) and
 * ad (fp32, [ffn/32]).  Returns 0, -1 on a bad shape, -2 on an expert id
 * out of range.                                                           */
int orc_expert_ffn(const orc_layer* L, int64_t ntok, const int8_t* xq,
                   const float* xd, const int32_t* idx, const float* wts,
                   double* y, double* g_out, double* u_out, int8_t* aq_out,
                   float* ad_out);

/* ---- shared expert ---------------------------------------------------------- */
/* The shared expert kept at higher precision beside the low-bit routed
 * experts (llama-modchip page, "The interesting bit": shared experts stay in
 * 4/5-bit or float formats while the routed experts go to 1-bit).  Reading:
 * 8-bit blocks of 32 weights (the Q8_0 layout of the pxq_llama tensor census,
 * "Full census"): per block d = fp16_RNE(amax / 127, in fp64) and
 * q = clamp(rint(w / d), -127, 127) (fp32 division by the fp16 value; a block
 * whose d is 0 is all zeros); stored row-major: q [rows][k] int8,
 * d [rows][k/32] fp16.  Its FFN output is added to every token's routed sum
 * with weight 1.                                                           */
int orc_quantize_weights_q8(const float* w, int64_t rows, int64_t k, int8_t* q,
                            uint16_t* d);
/* out[r] = sum_j d_w[r][j] * xd[j] * sum_{k in block j} q[r][k] * xq[k],
 * in fp64.                                                                */
void orc_matvec_q8(const int8_t* q, const uint16_t* d, int64_t rows, int64_t k,
                   const int8_t* xq, const float* xd, double* out);
/* y[t] += Wd_s . q8(silu(Wg_s . x^_t) * Wu_s . x^_t)^ for t < ntok (fp64),
 * gate/up [ffn][hidden], down [hidden][ffn], all in the q8 block format.
 * Returns 0, or -1 on a bad shape (hidden, ffn multiples of 32).          */
int orc_shared_ffn(int64_t hidden, int64_t ffn, const int8_t* gq, const uint16_t* gd,
                   const int8_t* uq, const uint16_t* ud, const int8_t* dq,
                   const uint16_t* dd, int64_t ntok, const int8_t* xq,
                   const float* xd, double* y);

#ifdef __cplusplus
}
#endif
#endif
