/*
 * moe_oracle.cpp -- CPU oracle for the MoE token-routing path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load, call or link this code.  The CUDA
 * library never uses it, and it shares no code, header, table or helper
 * with the CUDA library: the two are written independently so that a
 * disagreement between them means something.
 *
 * Plain, single-threaded, obviously-correct C++.  Floating-point softmax is
 * evaluated in double and rounded once to fp32; the combine accumulates in
 * fp32 with explicit fused multiply-adds (built with -ffp-contract=off so the
 * compiler cannot change the rounding anywhere else).
 *
 * Sources (web pages, by title and section):
 *   [UR]  "project_6/upstream_ref -- Upstream Reference: Deep-Spark xllm + vllm"
 *         sections "Call Chain: MoE topk_softmax on BI-V100" and "File Index".
 *   [CS]  "b70-optimization-lab: 2026-07-16 MTP1 M=2 compact scheduler closure
 *         note" -- the coverage paragraph, the scheduler paragraph and the
 *         route-pattern table.
 * Where the pages are silent the oracle takes one plain reading; every such
 * reading is named at the point where it is used ("reading: ...").
 *
 * Parity pins: every function here is pinned by CPU tests against closed
 * forms, brute force, hand-worked examples and invariants (tests/test_oracle_*.py).
 *
 * Return value of every entry point: 0 = OK, 1 = invalid argument.
 */
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

/* bf16 is the top half of an IEEE binary32; widening is exact. */
float bf16_to_float(uint16_t b) {
    uint32_t u = static_cast<uint32_t>(b) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 to bf16, round-to-nearest-even (NaN kept quiet). */
uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) {
        return static_cast<uint16_t>((u >> 16) | 0x0040u);
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return static_cast<uint16_t>(u >> 16);
}

double logit_as_double(const void* logits, int dtype, int64_t idx) {
    if (dtype == 1) {
        return static_cast<double>(bf16_to_float(static_cast<const uint16_t*>(logits)[idx]));
    }
    return static_cast<double>(static_cast<const float*>(logits)[idx]);
}

/* k rounds of "first maximum among the experts not yet taken": the largest logit, the lowest
 * expert index among equal logits (reading: lowest-index tie-break, selection made on the
 * logits themselves). */
void select_topk(const std::vector<double>& x, int32_t E, int32_t k, std::vector<char>& taken,
                 std::vector<int32_t>& sel) {
    for (int32_t e = 0; e < E; ++e) taken[e] = 0;
    for (int32_t j = 0; j < k; ++j) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || x[e] > x[best]) best = e; /* strict '>' keeps the lowest index */
        }
        taken[best] = 1;
        sel[j] = best;
    }
}

}  // namespace

extern "C" {

/*
 * Fused softmax + top-k gating of one row of router logits per token.
 * [UR] "File Index": moe_topk_softmax_kernels.cuh is the "fused softmax+topk"
 * kernel and topk_softmax_kernels.cu is vLLM's topk_softmax; "Call Chain: MoE
 * topk_softmax" places it between the router and the experts; the FusedMoE
 * layer listed there runs "gate -> topk -> expand -> ... -> combine".
 *
 * For every token t (row of E logits):
 *   1. select k experts, one at a time: the largest logit not yet taken, the
 *      lowest expert index among equal logits (reading: lowest-index
 *      tie-break, selection made on the logits themselves);
 *   2. m = max logit; Z = sum over all E experts of exp(x_e - m), summed in
 *      expert order, in double (reading: softmax over all E experts);
 *   3. weight_j = exp(x_sel_j - m) / Z, or / sum_j exp(x_sel_j - m) when
 *      renormalize != 0 (reading: renormalise in double, then round once);
 *   4. round the weight once to fp32; ids are stored in selection order.
 * dtype: 0 = fp32 logits, 1 = bf16 logits (as raw 16-bit patterns).
 */
int oracle_topk_softmax(const void* logits, int dtype, int64_t T, int32_t E, int32_t k,
                        int renormalize, float* topk_weights, int32_t* topk_ids) {
    if (T < 0 || E < 1 || k < 1 || k > E || (dtype != 0 && dtype != 1)) return 1;
    if (T > 0 && (logits == nullptr || topk_weights == nullptr || topk_ids == nullptr)) return 1;

    std::vector<double> x(static_cast<size_t>(E));
    std::vector<char> taken(static_cast<size_t>(E));
    std::vector<int32_t> sel(static_cast<size_t>(k));

    for (int64_t t = 0; t < T; ++t) {
        for (int32_t e = 0; e < E; ++e) x[e] = logit_as_double(logits, dtype, t * E + e);
        /* step 1: k rounds of "first maximum among the experts not yet taken" */
        select_topk(x, E, k, taken, sel);
        /* step 2: softmax denominator over all E experts */
        double m = x[0];
        for (int32_t e = 1; e < E; ++e) {
            if (x[e] > m) m = x[e];
        }
        double Z = 0.0;
        for (int32_t e = 0; e < E; ++e) Z += std::exp(x[e] - m);
        /* step 3: optional renormalisation over the k selected experts */
        double denom = Z;
        if (renormalize) {
            double S = 0.0;
            for (int32_t j = 0; j < k; ++j) S += std::exp(x[sel[j]] - m);
            denom = S;
        }
        /* step 4: one rounding to fp32 */
        for (int32_t j = 0; j < k; ++j) {
            double wj = std::exp(x[sel[j]] - m) / denom;
            topk_weights[t * k + j] = static_cast<float>(wj);
            topk_ids[t * k + j] = sel[j];
        }
    }
    return 0;
}

/*
 * Sigmoid scoring variant of the gating ("Upstream Reference: Deep-Spark xllm + vllm", "File
 * Index": moe_topk_sigmoid_kernels.cuh, "sigmoid variant for DeepSeek-style routing", chosen by
 * the sigmoid/softmax top-k dispatcher moe_fused_topk.cu).  The page gives no formula; the
 * plainest reading, taken here:
 *   1. select k experts exactly as oracle_topk_softmax does (on the logits; the logistic
 *      function is increasing, so this is also the order of the scores);
 *   2. score_j = 1 / (1 + exp(-x_sel_j)) in double, each expert on its own (no normalisation
 *      across experts);
 *   3. weight_j = score_j, or score_j / sum_j score_j when renormalize != 0 (1/k when that sum
 *      is 0, which needs every selected logit below about -745);
 *   4. round the weight once to fp32; ids are stored in selection order.
 */
int oracle_topk_sigmoid(const void* logits, int dtype, int64_t T, int32_t E, int32_t k,
                        int renormalize, float* topk_weights, int32_t* topk_ids) {
    if (T < 0 || E < 1 || k < 1 || k > E || (dtype != 0 && dtype != 1)) return 1;
    if (T > 0 && (logits == nullptr || topk_weights == nullptr || topk_ids == nullptr)) return 1;

    std::vector<double> x(static_cast<size_t>(E));
    std::vector<char> taken(static_cast<size_t>(E));
    std::vector<int32_t> sel(static_cast<size_t>(k));
    std::vector<double> score(static_cast<size_t>(k));

    for (int64_t t = 0; t < T; ++t) {
        for (int32_t e = 0; e < E; ++e) x[e] = logit_as_double(logits, dtype, t * E + e);
        select_topk(x, E, k, taken, sel);
        double S = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            score[j] = 1.0 / (1.0 + std::exp(-x[sel[j]]));
            S += score[j];
        }
        for (int32_t j = 0; j < k; ++j) {
            const double wj = renormalize ? (S > 0.0 ? score[j] / S : 1.0 / k) : score[j];
            topk_weights[t * k + j] = static_cast<float>(wj);
            topk_ids[t * k + j] = sel[j];
        }
    }
    return 0;
}

/* Rows of the block-padded expert-grouped layout: C = T*k + E_local*(block_size-1),
 * the largest possible padded total (every local expert wastes < block_size rows). */
int64_t oracle_align_capacity(int64_t T, int32_t k, int32_t E_local, int32_t block_size) {
    if (T < 0 || k < 1 || E_local < 1 || block_size < 1) return -1;
    return T * k + static_cast<int64_t>(E_local) * (block_size - 1);
}

/*
 * Per-expert histogram, block-padded prefix and stable placement of the
 * routed slots, with the expert-parallel remap.
 * [UR] "File Index": moe_align_sum_kernels.cu does "block alignment for
 * scatter".  [CS] scheduler paragraph: each local expert's row count and
 * remapped-row prefix are derived from topk_ids plus expert_map, and in the
 * all-duplicate case occurrence 0 and occurrence 8 own the two 8-row tiles;
 * [CS] coverage paragraph: an all-remote expert-parallel rank is valid.
 *
 * Slot s = t*k + j.  Its local expert is le = expert_map[topk_ids[s]] (or the
 * id itself when expert_map is NULL, which needs E_local == E_global).  A slot
 * is remote (dropped) when le < 0; an id outside [0, E_global) or a mapped
 * value outside [-1, E_local) is also treated as remote (reading).
 *   counts[e]   = number of local slots on expert e
 *   offsets[e]  = exclusive prefix of ceil(counts/bs)*bs;  offsets[E_local] = N_pad
 *   rows offsets[e] .. offsets[e]+counts[e]-1 hold the slots of expert e in
 *   ascending s (stable by expert, token, slot); the rest of the expert's
 *   padded range and every row from N_pad to capacity hold the pad value T*k
 *   inv_perm[s] = row of slot s, or -1 for a remote slot
 *   expert_ids[b] = expert of block b, -1 for blocks at or past N_pad/bs
 * Output sizes: counts[E_local], offsets[E_local+1], sorted_token_ids[C],
 * expert_ids[ceil(C/bs)], num_tokens_post_pad[1], inv_perm[T*k].
 */
int oracle_align_permute(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E_global,
                         const int32_t* expert_map, int32_t E_local, int32_t block_size,
                         int32_t* counts, int32_t* offsets, int32_t* sorted_token_ids,
                         int32_t* expert_ids, int32_t* num_tokens_post_pad, int32_t* inv_perm) {
    if (T < 0 || k < 1 || E_global < 1 || E_local < 1 || block_size < 1) return 1;
    if (expert_map == nullptr && E_local != E_global) return 1;
    if (E_local > E_global) return 1;
    const int64_t P = T * k;
    const int64_t C = oracle_align_capacity(T, k, E_local, block_size);
    const int64_t NB = (C + block_size - 1) / block_size;

    std::vector<std::vector<int64_t>> rows_of(static_cast<size_t>(E_local));
    for (int64_t s = 0; s < P; ++s) {
        int32_t g = topk_ids[s];
        int32_t le = -1;
        if (g >= 0 && g < E_global) le = (expert_map != nullptr) ? expert_map[g] : g;
        if (le >= E_local) le = -1;
        if (le >= 0) rows_of[le].push_back(s); /* ascending s: the stable order */
    }

    int64_t running = 0;
    for (int32_t e = 0; e < E_local; ++e) {
        int64_t n = static_cast<int64_t>(rows_of[e].size());
        int64_t padded = ((n + block_size - 1) / block_size) * block_size;
        counts[e] = static_cast<int32_t>(n);
        offsets[e] = static_cast<int32_t>(running);
        running += padded;
    }
    offsets[E_local] = static_cast<int32_t>(running);
    num_tokens_post_pad[0] = static_cast<int32_t>(running);

    for (int64_t p = 0; p < C; ++p) sorted_token_ids[p] = static_cast<int32_t>(P);
    for (int64_t s = 0; s < P; ++s) inv_perm[s] = -1;
    for (int32_t e = 0; e < E_local; ++e) {
        for (size_t i = 0; i < rows_of[e].size(); ++i) {
            int64_t row = offsets[e] + static_cast<int64_t>(i);
            sorted_token_ids[row] = static_cast<int32_t>(rows_of[e][i]);
            inv_perm[rows_of[e][i]] = static_cast<int32_t>(row);
        }
    }

    for (int64_t b = 0; b < NB; ++b) expert_ids[b] = -1;
    for (int32_t e = 0; e < E_local; ++e) {
        for (int64_t b = offsets[e] / block_size; b < offsets[e + 1] / block_size; ++b) {
            expert_ids[b] = e;
        }
    }
    return 0;
}

/*
 * Activation permute-gather ("expand" in the FusedMoE pipeline of [UR]
 * "File Index"; "direct slot-order gather" in [CS]).  Walks the rows of the
 * expert-grouped layout in order: row p < N_pad that holds slot s receives a
 * bit copy of hidden[s / k]; a pad row is left untouched, or set to +0 when
 * zero_pad != 0.  Rows at or past N_pad are never written.
 */
int oracle_gather(const uint16_t* hidden, int64_t T, int32_t H, int32_t k,
                  const int32_t* sorted_token_ids, int32_t num_tokens_post_pad, int zero_pad,
                  uint16_t* permuted) {
    if (T < 0 || H < 1 || k < 1 || num_tokens_post_pad < 0) return 1;
    const int64_t P = T * k;
    for (int64_t p = 0; p < num_tokens_post_pad; ++p) {
        int64_t s = sorted_token_ids[p];
        uint16_t* dst = permuted + p * H;
        if (s >= 0 && s < P) {
            std::memcpy(dst, hidden + (s / k) * H, sizeof(uint16_t) * static_cast<size_t>(H));
        } else if (zero_pad) {
            std::memset(dst, 0, sizeof(uint16_t) * static_cast<size_t>(H));
        }
    }
    return 0;
}

/*
 * Top-k weighted combine back to token order ("combine" in the FusedMoE
 * pipeline of [UR] "File Index"; the "sum" in moe_align_sum_kernels.cu).
 *   out[t, h] = bf16_rne( acc ),  acc = +0.0f, then for j = 0 .. k-1 with
 *   r = inv_perm[t*k + j] >= 0:  acc = fmaf(w[t, j], float(y[r, h]), acc).
 * fp32 accumulation follows the "full fp32 accumulation" lesson of the GDN
 * call chain in [UR]; the fixed ascending-j order and the explicit fused
 * multiply-add are a reading.  Remote slots (-1) contribute nothing, so an
 * all-remote token gets +0 (the expert-parallel partial sum).
 */
int oracle_combine(const uint16_t* expert_out, const float* topk_weights, const int32_t* inv_perm,
                   int64_t T, int32_t k, int32_t H, uint16_t* out) {
    if (T < 0 || k < 1 || H < 1) return 1;
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                int64_t r = inv_perm[t * k + j];
                if (r < 0) continue;
                float y = bf16_to_float(expert_out[r * H + h]);
                acc = std::fma(topk_weights[t * k + j], y, acc);
            }
            out[t * H + h] = float_to_bf16_rne(acc);
        }
    }
    return 0;
}

/* The exchange after an expert-parallel combine: each of n ranks holds a bf16 partial [rows, H] (the
 * combine over its local slots, remote slots dropped); the layer output is the sum of the partials.
 * Reading (the closure note leaves the collective out): widened to fp32, summed in ascending rank
 * order starting from +0, rounded once to bf16.  partials: [n][rows][H] bf16 bits, rank-major. */
int oracle_reduce_partials(const uint16_t* partials, int32_t n, int64_t rows, int32_t H, uint16_t* out) {
    if (n < 1 || rows < 0 || H < 1) return 1;
    const int64_t m = rows * static_cast<int64_t>(H);
    for (int64_t i = 0; i < m; ++i) {
        float acc = 0.0f;
        for (int32_t r = 0; r < n; ++r) acc = acc + bf16_to_float(partials[r * m + i]);
        out[i] = float_to_bf16_rne(acc);
    }
    return 0;
}

}  // extern "C"
