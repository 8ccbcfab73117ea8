/*
 * Plain CPU oracle for rank-major MoE expert-parallel dispatch and combine.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only the test suite, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header or table with the CUDA library.
 *
 * Every function is the plain definition of what the method computes, written
 * as nested loops in the order "source rank -> token -> top_k slot", with no
 * blocking, fusion or reordering.  All virtual ranks live in one address space,
 * so a "send" is a memcpy into the destination rank's receive array.
 *
 * Notation (pages' names):
 *   ep_size            number of expert-parallel ranks
 *   num_experts (E)    global expert count; experts_per_rank = E / ep_size
 *   top_k (k)          experts selected per token
 *   tokens_per_rank    the step's runtime_max_tokens_per_rank (tpr)
 *   local_num_tokens   n[r], tokens rank r holds this step, n[r] <= tpr
 *
 * Sources:
 *   [OSC]  flashinfer.moe_ep.NVLinkOneSidedConfig, `lamport` paragraph: rows a
 *          rank receives from rank src for token t land at
 *          src * tokens_per_rank + t.
 *   [TSD]  flashinfer.moe_ep.NVLinkTwoSidedAlltoAll, dispatch(): a token goes to
 *          every rank owning one of the experts chosen for it; topk_ids hold
 *          global expert ids; weights and scales move in the token's row slot.
 *   [TSC]  same page, combine(): each rank returns one row per token, its own
 *          experts' outputs weighted and summed; the rows are summed over ranks.
 *   [A2A]  flashinfer.comm.moe_a2a_dispatch, Parameters (active_rank_mask,
 *          eplb_local_stats) and Returns (eplb_gathered_stats row r = rank r).
 *   [V2S]  vllm.distributed.device_communicators.all2all,
 *          FlashInferNVLinkTwoSidedManager.get_communication: a received row
 *          beyond a source's tokens carries the id num_experts.
 *   [OSCu] flashinfer.moe_ep.NVLinkOneSidedConfig, `use_low_precision_combine`:
 *          combine payloads travel as FP8.
 *   [AGRS] vllm.distributed.device_communicators.all2all, AgRsAll2AllManager:
 *          dispatch as an all-gather of every rank's rows, combine as a
 *          reduce-scatter (each rank gets its own rows summed over all ranks).
 *   [TSCi] flashinfer.moe_ep.NVLinkTwoSidedAlltoAll, combine(): its input rows
 *          come out of a per-rank weighting and summing over the rank's own
 *          experts; oracle_expert_reduce states that step.
 *
 * Readings where the pages are silent (each is one deliberate choice):
 *   - expert e is owned by rank e / (E / ep_size) (contiguous blocks);
 *   - an id outside [0, E) is owned by no rank and is not routed;
 *   - a token reaches each owning rank once, however many of its experts that
 *     rank owns (the slot src*tpr+t is unique per token);
 *   - one active_rank_mask is shared by all virtual ranks; a rank whose bit is
 *     clear neither sends nor receives; its receive arrays are left untouched;
 *   - the combine sum is an fp32 accumulator starting at +0.0f, adding the rows
 *     in ascending destination-rank order, rounded once to bf16 (nearest-even);
 *   - the FP8 combine format is E4M3 ("fn": no infinities, max 448), unscaled,
 *     or, in the scaled variant, E4M3 with one fp32 scale per row: with
 *     amax = max |x| over the row, scale = amax / 448 and the codes are
 *     E4M3(x * (448 / amax)) (each fp32 operation rounded to nearest); a zero
 *     row has scale 1; the combine adds fmaf(decode(q), scale, acc);
 *   - expert outputs before that reduction are one BF16 row per (source token,
 *     top_k slot), [ep, tpr, k, hidden]; rank d's combine row for the token is
 *     bf16(sum over the slots j whose expert d owns, ascending j, of
 *     w_j * y_j), each term added with one fused multiply-add (fmaf) to an fp32
 *     accumulator that starts at +0.0f.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Number formats, from their definitions.                                   */
/* ------------------------------------------------------------------------- */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* bf16 is the upper half of an fp32 word: widening is exact. */
float oracle_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even, on the 16 dropped bits.
 * A carry out of the mantissa moves into the exponent, which is exactly
 * rounding up to the next binade (or to infinity past the largest finite).
 * NaN stays NaN (quiet bit set, sign kept). */
uint16_t oracle_bf16_from_f32(float f) {
    uint32_t u = f32_bits(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; there is no
 * infinity, the largest finite magnitude is 1.75 * 2^8 = 448. */
float oracle_e4m3_to_f32(uint8_t b) {
    int s = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 7;
    double v;
    if (e == 15 && m == 7) return s ? -NAN : NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* fp32 -> E4M3, round to nearest, ties to even, saturating to +-448 (also for
 * infinities).  The magnitude is scaled so that its 3 fraction bits become the
 * integer part, rounded with rint() (the default rounding mode is nearest-even)
 * and scaled back; below 2^-6 the spacing is the subnormal step 2^-9. */
uint8_t oracle_e4m3_from_f32(float f) {
    if (isnan(f)) return 0x7F;
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);             /* a = fr * 2^ex, fr in [0.5, 1) */
    int e = ex - 1;            /* a in [2^e, 2^(e+1)) */
    if (e < -6) e = -6;        /* subnormal range shares the 2^-6 binade's spacing */
    double step = ldexp(1.0, e - 3);
    double q = rint(a / step); /* integer count of steps, ties to even */
    double r = q * step;
    if (r >= 448.0) return sign | 0x7E;   /* 448 is representable; only saturates */
    if (r == 0.0) return sign;
    /* encode r exactly */
    frexp(r, &ex);
    e = ex - 1;
    if (e < -6) {              /* subnormal: r = m * 2^-9 */
        int m = (int)ldexp(r, 9);
        return sign | (uint8_t)m;
    }
    int m = (int)ldexp(r, 3 - e) - 8;  /* r = (1 + m/8) * 2^e */
    return sign | (uint8_t)(((e + 7) << 3) | m);
}

void oracle_quantize_e4m3(const uint16_t* bf16_in, uint8_t* e4m3_out, int64_t n) {
    for (int64_t i = 0; i < n; ++i)
        e4m3_out[i] = oracle_e4m3_from_f32(oracle_bf16_to_f32(bf16_in[i]));
}

/* ------------------------------------------------------------------------- */
/* Routing plan.                                                             */
/* ------------------------------------------------------------------------- */

static int rank_is_live(const uint64_t* active_rank_mask, int r) {
    if (active_rank_mask == 0) return 1;
    return (int)((active_rank_mask[r / 64] >> (r % 64)) & 1u);
}

/*
 * For every live source rank r and token t < n[r]: the destination set is the
 * set of live ranks owning any of the token's k experts [TSD], listed in
 * ascending rank order.  num_dst[r][t] is its size; dst_ranks[r][t][0..k) holds
 * it, padded with -1.  Tokens that do not exist (t >= n[r], or r masked off)
 * get num_dst = -1.
 *
 * For every live destination d and every slot s = r*tpr + t [OSC]:
 *   recv_valid[d][s]     = 1 if d is in the token's destination set, else 0;
 *   recv_topk_ids[d][s]  = the token's k global ids verbatim when valid [TSD],
 *                          else invalid_expert_id in all k entries [V2S].
 * Rows of masked-off destinations are not written [A2A: such a rank does not
 * take part].
 * send_counts[r][d] = number of tokens of r whose set contains d (all ep*ep
 * entries written).
 */
int oracle_route(int ep_size, int num_experts, int top_k, int tokens_per_rank,
                 const int32_t* token_selected_experts, /* [ep, tpr, k] */
                 const int32_t* local_num_tokens,       /* [ep] */
                 const uint64_t* active_rank_mask,      /* words or NULL */
                 int32_t invalid_expert_id,
                 int32_t* num_dst,        /* [ep, tpr] */
                 int32_t* dst_ranks,      /* [ep, tpr, k] */
                 int32_t* send_counts,    /* [ep, ep] */
                 uint8_t* recv_valid,     /* [ep, ep*tpr] */
                 int32_t* recv_topk_ids)  /* [ep, ep*tpr, k] */
{
    const int ep = ep_size, k = top_k, tpr = tokens_per_rank;
    if (ep <= 0 || num_experts % ep != 0) return -1;
    const int experts_per_rank = num_experts / ep;
    const int64_t slots = (int64_t)ep * tpr;
    unsigned char seen[1024];
    if (ep > 1024) return -1;

    for (int r = 0; r < ep; ++r)
        for (int d = 0; d < ep; ++d) send_counts[r * ep + d] = 0;

    /* every slot of every live destination starts invalid */
    for (int d = 0; d < ep; ++d) {
        if (!rank_is_live(active_rank_mask, d)) continue;
        for (int64_t s = 0; s < slots; ++s) {
            recv_valid[d * slots + s] = 0;
            for (int j = 0; j < k; ++j)
                recv_topk_ids[(d * slots + s) * k + j] = invalid_expert_id;
        }
    }

    for (int r = 0; r < ep; ++r) {
        const int live_r = rank_is_live(active_rank_mask, r);
        for (int t = 0; t < tpr; ++t) {
            int32_t* list = dst_ranks + ((int64_t)r * tpr + t) * k;
            for (int j = 0; j < k; ++j) list[j] = -1;
            if (!live_r || t >= local_num_tokens[r]) {
                num_dst[r * tpr + t] = -1;
                continue;
            }
            const int32_t* ids = token_selected_experts + ((int64_t)r * tpr + t) * k;
            memset(seen, 0, (size_t)ep);
            for (int j = 0; j < k; ++j) {
                int32_t e = ids[j];
                if (e < 0 || e >= num_experts) continue;     /* owned by no rank */
                int owner = e / experts_per_rank;
                if (!rank_is_live(active_rank_mask, owner)) continue; /* dropped */
                seen[owner] = 1;
            }
            int nd = 0;
            for (int d = 0; d < ep; ++d) {
                if (!seen[d]) continue;
                list[nd++] = d;
                const int64_t s = (int64_t)r * tpr + t;
                recv_valid[d * slots + s] = 1;
                for (int j = 0; j < k; ++j)
                    recv_topk_ids[(d * slots + s) * k + j] = ids[j];
                send_counts[r * ep + d] += 1;
            }
            num_dst[r * tpr + t] = nd;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Dispatch of one payload.                                                   */
/* ------------------------------------------------------------------------- */

/*
 * recv[d][r*tpr + t][:] = in[r][t][:] for every d in the token's destination
 * set [OSC, TSD].  Bytes are copied verbatim; rows of invalid slots are left as
 * they were.  only_dst >= 0 restricts the copy to that destination (the same
 * loop, with the other destinations skipped), so that large cases can be
 * checked one receive array at a time.
 */
void oracle_dispatch_payload(int ep_size, int top_k, int tokens_per_rank,
                             int64_t row_bytes,
                             const uint8_t* in,        /* [ep, tpr, row_bytes] */
                             const int32_t* num_dst,   /* [ep, tpr] */
                             const int32_t* dst_ranks, /* [ep, tpr, k] */
                             uint8_t* recv,            /* [ep or 1, ep*tpr, row_bytes] */
                             int only_dst)
{
    const int ep = ep_size, k = top_k, tpr = tokens_per_rank;
    const int64_t slots = (int64_t)ep * tpr;
    for (int r = 0; r < ep; ++r) {
        for (int t = 0; t < tpr; ++t) {
            const int nd = num_dst[r * tpr + t];
            const int32_t* list = dst_ranks + ((int64_t)r * tpr + t) * k;
            for (int i = 0; i < nd; ++i) {
                const int d = list[i];
                if (only_dst >= 0 && d != only_dst) continue;
                const int64_t s = (int64_t)r * tpr + t;
                uint8_t* dst = recv + ((only_dst >= 0 ? 0 : (int64_t)d) * slots + s) * row_bytes;
                const uint8_t* src = in + ((int64_t)r * tpr + t) * row_bytes;
                memcpy(dst, src, (size_t)row_bytes);
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* EPLB statistics gather.                                                    */
/* ------------------------------------------------------------------------- */

/*
 * Every live destination d receives row r = rank r's local statistics [A2A,
 * Returns].  A masked-off source contributes a zero row (reading: it takes no
 * part in the step).  Masked-off destinations are not written.
 */
void oracle_eplb_gather(int ep_size, int num_stats,
                        const int32_t* eplb_local_stats, /* [ep, num_stats] */
                        const uint64_t* active_rank_mask,
                        int32_t* eplb_gathered_stats)    /* [ep, ep, num_stats] */
{
    const int ep = ep_size;
    for (int d = 0; d < ep; ++d) {
        if (!rank_is_live(active_rank_mask, d)) continue;
        for (int r = 0; r < ep; ++r) {
            const int live_r = rank_is_live(active_rank_mask, r);
            for (int e = 0; e < num_stats; ++e)
                eplb_gathered_stats[((int64_t)d * ep + r) * num_stats + e] =
                    live_r ? eplb_local_stats[(int64_t)r * num_stats + e] : 0;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Combine.                                                                   */
/* ------------------------------------------------------------------------- */

/*
 * For a token (r, t) that exists, and every hidden column h:
 *   acc = +0.0f;  for d in the destination set, ascending:
 *       acc = acc + float(expert_output[d][r*tpr + t][h])   (one fp32 add)
 *   out[r][t][h] = bf16_round_nearest_even(acc)
 * [TSC; OSCu for the E4M3 input].  A token whose destination set is empty
 * (all owners masked off) combines to +0.0.  Rows of tokens that do not exist
 * are left as they were.  Only rows of valid slots are read.
 *
 * token_list (length n_list, entries r*tpr+t) restricts the work to those
 * tokens; NULL means all tokens.
 */
void oracle_combine(int ep_size, int top_k, int tokens_per_rank, int hidden,
                    const int32_t* num_dst, const int32_t* dst_ranks,
                    const void* expert_output, /* [ep, ep*tpr, hidden] bf16 or e4m3 */
                    int input_is_e4m3,
                    uint16_t* out,             /* [ep, tpr, hidden] bf16 */
                    const int64_t* token_list, int64_t n_list)
{
    const int ep = ep_size, k = top_k, tpr = tokens_per_rank;
    const int64_t slots = (int64_t)ep * tpr;
    const int64_t n_tokens = token_list ? n_list : slots;
    for (int64_t i = 0; i < n_tokens; ++i) {
        const int64_t s = token_list ? token_list[i] : i;   /* s = r*tpr + t */
        const int nd = num_dst[s];
        if (nd < 0) continue;
        const int32_t* list = dst_ranks + s * k;
        for (int h = 0; h < hidden; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < nd; ++j) {
                const int d = list[j];
                const int64_t idx = ((int64_t)d * slots + s) * hidden + h;
                float x;
                if (input_is_e4m3) x = oracle_e4m3_to_f32(((const uint8_t*)expert_output)[idx]);
                else x = oracle_bf16_to_f32(((const uint16_t*)expert_output)[idx]);
                acc = acc + x;
            }
            out[s * hidden + h] = oracle_bf16_from_f32(acc);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Weighted reduction over each rank's local experts (the combine's input).  */
/* ------------------------------------------------------------------------- */

/*
 * For a token (r, t) that exists and every rank d in its destination set,
 * rank d's combine row [TSCi] is
 *   z[d][r*tpr + t][h] = bf16( sum over j ascending with owner(ids[j]) == d of
 *                              w[r][t][j] * y[r][t][j][h] )
 * where the sum is an fp32 accumulator starting at +0.0f and each term is one
 * fmaf (product and add rounded once).  Slots whose expert is owned by no rank
 * or by a masked-off rank are not in any destination's sum.  Rows of z that no
 * token fills are left as they were.  Feeding z to oracle_combine gives the
 * combine of the per-expert outputs.
 */
void oracle_expert_reduce(int ep_size, int num_experts, int top_k, int tokens_per_rank,
                          int hidden, const int32_t* num_dst, const int32_t* dst_ranks,
                          const int32_t* token_selected_experts, /* [ep, tpr, k] */
                          const float* topk_weights,             /* [ep, tpr, k] */
                          const uint16_t* expert_out,            /* [ep, tpr, k, hidden] */
                          uint16_t* z)                           /* [ep, ep*tpr, hidden] */
{
    const int ep = ep_size, k = top_k, tpr = tokens_per_rank;
    const int experts_per_rank = num_experts / ep;
    const int64_t slots = (int64_t)ep * tpr;
    for (int64_t s = 0; s < slots; ++s) {
        const int nd = num_dst[s];
        const int32_t* ids = token_selected_experts + s * k;
        const float* w = topk_weights + s * k;
        for (int i = 0; i < nd; ++i) {
            const int d = dst_ranks[s * k + i];
            for (int h = 0; h < hidden; ++h) {
                float acc = 0.0f;
                for (int j = 0; j < k; ++j) {
                    const int32_t e = ids[j];
                    if (e < 0 || e >= num_experts || e / experts_per_rank != d) continue;
                    const float y = oracle_bf16_to_f32(expert_out[(s * k + j) * hidden + h]);
                    acc = fmaf(w[j], y, acc);
                }
                z[((int64_t)d * slots + s) * hidden + h] = oracle_bf16_from_f32(acc);
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* FP8 combine with one scale per row.                                        */
/* ------------------------------------------------------------------------- */

/*
 * Per row of `hidden` bf16 values: amax = max |x|; scale = amax / 448 and
 * inv = 448 / amax, each an fp32 division rounded to nearest (1 and 1 for a
 * zero row); code[h] = E4M3(x[h] * inv) with the product rounded to fp32 and
 * the E4M3 rounding of oracle_e4m3_from_f32 (nearest even, saturating).
 */
void oracle_quantize_e4m3_rows(const uint16_t* bf16_in, int64_t rows, int hidden,
                               uint8_t* e4m3_out, float* scales) {
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* x = bf16_in + r * hidden;
        float amax = 0.0f;
        for (int h = 0; h < hidden; ++h) {
            const float a = fabsf(oracle_bf16_to_f32(x[h]));
            if (a > amax) amax = a;
        }
        float scale = 1.0f, inv = 1.0f;
        if (amax > 0.0f) {
            scale = amax / 448.0f;
            inv = 448.0f / amax;
        }
        scales[r] = scale;
        for (int h = 0; h < hidden; ++h) {
            const float v = oracle_bf16_to_f32(x[h]) * inv;
            e4m3_out[r * hidden + h] = oracle_e4m3_from_f32(v);
        }
    }
}

/*
 * As oracle_combine with E4M3 rows, each destination row carrying its scale
 * (row_scales [ep(dst), ep*tpr]):  acc = fmaf(decode(q), scale, acc) for d in
 * the token's destination set, ascending, from +0.0f; out = bf16(acc).
 */
void oracle_combine_scaled(int ep_size, int top_k, int tokens_per_rank, int hidden,
                           const int32_t* num_dst, const int32_t* dst_ranks,
                           const uint8_t* expert_output, const float* row_scales,
                           uint16_t* out)
{
    const int ep = ep_size, k = top_k, tpr = tokens_per_rank;
    const int64_t slots = (int64_t)ep * tpr;
    for (int64_t s = 0; s < slots; ++s) {
        const int nd = num_dst[s];
        if (nd < 0) continue;
        const int32_t* list = dst_ranks + s * k;
        for (int h = 0; h < hidden; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < nd; ++j) {
                const int d = list[j];
                const int64_t row = (int64_t)d * slots + s;
                acc = fmaf(oracle_e4m3_to_f32(expert_output[row * hidden + h]), row_scales[row], acc);
            }
            out[s * hidden + h] = oracle_bf16_from_f32(acc);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Dense variant [AGRS]: every rank gets every token; every rank's row sums.  */
/* ------------------------------------------------------------------------- */

/*
 * Every live rank receives every token of every live source rank:
 * recv[d][r*tpr + t] = in[r][t] for live d, live r, t < n[r].  Other rows
 * are left as they were.  (The rank-major slot layout is kept, so that the
 * two variants read and write the same arrays.)
 */
void oracle_allgather(int ep_size, int tokens_per_rank, int64_t row_bytes,
                      const int32_t* local_num_tokens, const uint64_t* active_rank_mask,
                      const uint8_t* in, uint8_t* recv)
{
    const int ep = ep_size, tpr = tokens_per_rank;
    const int64_t slots = (int64_t)ep * tpr;
    for (int r = 0; r < ep; ++r) {
        if (!rank_is_live(active_rank_mask, r)) continue;
        for (int t = 0; t < local_num_tokens[r]; ++t) {
            const int64_t s = (int64_t)r * tpr + t;
            for (int d = 0; d < ep; ++d) {
                if (!rank_is_live(active_rank_mask, d)) continue;
                memcpy(recv + ((int64_t)d * slots + s) * row_bytes, in + s * row_bytes,
                       (size_t)row_bytes);
            }
        }
    }
}

/*
 * out[r][t][h] = bf16( fp32 sum over live ranks d, ascending, from +0.0f, of
 * x[d][r*tpr + t][h] ) for live r, t < n[r]; other rows are left as they were.
 */
void oracle_reduce_scatter(int ep_size, int tokens_per_rank, int hidden,
                           const int32_t* local_num_tokens, const uint64_t* active_rank_mask,
                           const uint16_t* x, uint16_t* out)
{
    const int ep = ep_size, tpr = tokens_per_rank;
    const int64_t slots = (int64_t)ep * tpr;
    for (int r = 0; r < ep; ++r) {
        if (!rank_is_live(active_rank_mask, r)) continue;
        for (int t = 0; t < local_num_tokens[r]; ++t) {
            const int64_t s = (int64_t)r * tpr + t;
            for (int h = 0; h < hidden; ++h) {
                float acc = 0.0f;
                for (int d = 0; d < ep; ++d) {
                    if (!rank_is_live(active_rank_mask, d)) continue;
                    acc = acc + oracle_bf16_to_f32(x[((int64_t)d * slots + s) * hidden + h]);
                }
                out[s * hidden + h] = oracle_bf16_from_f32(acc);
            }
        }
    }
}
