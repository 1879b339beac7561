// fp64 CPU oracle for the H3-style DiT self-attention core.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
// this file: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
// reference arm do.  It shares no code, header, table or constant generator with
// the CUDA library; both sides only receive the same seeded input arrays.
//
// What it states, each function citing the passage it follows:
//   * QK-RMSNorm followed by 3D RoPE, fused and lossless (the fusion leaves the
//     results unchanged): news.cocoloop.cn, MiniMax-H3 SGLang report, section "Erst drei
//     übereinandergelegte Beschleunigungsebenen", fused-operator paragraph.
//     The 3D multimodal RoPE and the head geometry (hidden 5376 / 56 heads = 96)
//     come from 52hbtv.com, H3-Image port, section 二, model table.
//   * Blockwise KV-block router at sparsity 0.75 / 0.80 (same cocoloop page,
//     SubBlock paragraph); pooling, scoring and selection are fixed by the
//     problem statement: mean-pooled 128-token blocks, fp32 block scores,
//     per-query-block top-k, ties to the lower block index.
//   * Dense lossless attention (cocoloop page, opening quote: the dense path
//     approximates nothing) and block-sparse attention over the routed KV blocks,
//     bidirectional (cocoloop page, "Ein paar Grenzen": non-causal).
//   * The other operators the fused-operator paragraph of the cocoloop page
//     names -- the AdaLN update, the gated residual path and the SwiGLU
//     activation -- with their usual DiT definitions (the page gives none):
//     h = x + gate * f, y = LayerNorm(h) * (1 + scale) + shift with no affine
//     LayerNorm, and silu(a) * b.
//   * The Cache-DiT reuse decision (same page, the paragraph after it): a
//     residual-difference threshold, 0.04 conservative or 0.08 in stride mode,
//     decides whether a step's result is reused; read as the relative L1
//     difference sum|cur - prev| / sum|prev| of two steps' residuals.
//
// Everything is computed in double precision from the bf16 input bits, with
// plain loops and no blocking, fusion or reordering beyond the definitions.
// Readings where the pages are silent (pairing, token order, tail block, ...)
// are listed in the repository's design notes.

#include <algorithm>
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

double bf16_to_double(uint16_t bits) {
    uint32_t u = static_cast<uint32_t>(bits) << 16;
    float f;
    std::memcpy(&f, &u, sizeof(f));
    return static_cast<double>(f);
}

// Round a double to the nearest bf16 (8 significant bits, fp32 exponent
// range), ties to even, directly from double (no intermediate fp32 rounding).
uint16_t double_to_bf16_rne(double x) {
    if (std::isnan(x)) return 0x7FC0;
    double r;
    const double ax = std::fabs(x);
    if (ax == 0.0) {
        r = x;
    } else if (ax < std::ldexp(1.0, -126)) {  // subnormal range: fixed step 2^-133
        r = std::nearbyint(std::ldexp(x, 133)) * std::ldexp(1.0, -133);
    } else {
        int e;
        std::frexp(ax, &e);  // ax in [2^(e-1), 2^e)
        r = std::nearbyint(std::ldexp(x, 8 - e)) * std::ldexp(1.0, e - 8);
    }
    if (std::fabs(r) > 3.3895313892515355e38) r = std::copysign(INFINITY, x);  // beyond bf16 max
    float f = static_cast<float>(r);  // exact: r has at most 8 significant bits
    uint32_t u;
    std::memcpy(&u, &f, sizeof(u));
    return static_cast<uint16_t>(u >> 16);
}

int pick_threads(int nthreads) {
    if (nthreads > 0) return nthreads;
    unsigned hc = std::thread::hardware_concurrency();
    return hc == 0 ? 1 : static_cast<int>(hc);
}

// Run body(i) for i in [0, n) on up to nthreads threads (static interleave).
template <class F>
void parallel_for(int64_t n, int nthreads, F body) {
    int nt = pick_threads(nthreads);
    if (nt > n) nt = static_cast<int>(n > 0 ? n : 1);
    if (nt <= 1) {
        for (int64_t i = 0; i < n; ++i) body(i);
        return;
    }
    std::vector<std::thread> pool;
    pool.reserve(nt);
    for (int t = 0; t < nt; ++t) {
        pool.emplace_back([=, &body]() {
            for (int64_t i = t; i < n; i += nt) body(i);
        });
    }
    for (auto& th : pool) th.join();
}

// Element (b, n, h, c) of a contiguous [B, N, heads, d] tensor.
inline int64_t bshd_index(int b, int64_t n, int h, int c, int64_t N, int heads, int d) {
    return ((static_cast<int64_t>(b) * N + n) * heads + h) * d + c;
}

}  // namespace

extern "C" {

int oracle_abi_version() { return 1; }

int oracle_threads(int nthreads) { return pick_threads(nthreads); }

// bf16 bit pattern -> value (exact widening).
double oracle_bf16_to_double(uint16_t bits) { return bf16_to_double(bits); }

// RMSNorm of one head vector (cocoloop report, fused "QK-RMSNorm"):
//   y_i = x_i / sqrt(mean_j x_j^2 + eps) * gamma_i
void oracle_rmsnorm(const double* x, int d, const double* gamma, double eps, double* y) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double inv = 1.0 / std::sqrt(ss / d + eps);
    for (int i = 0; i < d; ++i) y[i] = x[i] * inv * gamma[i];
}

// 3D RoPE of one head vector in place (52hbtv page, "3D multimodal RoPE").
// The head dimension is split into three equal sections, one per grid axis
// (t, h, w in that order).  Inside section a, channels (2j, 2j+1) form the
// j-th rotation pair and turn by angle pos[a] * theta^(-2j / section_width).
// Requires d divisible by 6.
void oracle_rope3d(double* y, int d, const int* pos, double theta) {
    const int sec = d / 3;
    for (int a = 0; a < 3; ++a) {
        for (int j = 0; j < sec / 2; ++j) {
            double inv_freq = std::pow(theta, -2.0 * j / sec);
            double ang = pos[a] * inv_freq;
            double c = std::cos(ang), s = std::sin(ang);
            int i0 = a * sec + 2 * j, i1 = i0 + 1;
            double y0 = y[i0], y1 = y[i1];
            y[i0] = y0 * c - y1 * s;
            y[i1] = y0 * s + y1 * c;
        }
    }
}

// Grid position of flattened token n on a (T, H, W) grid, row-major:
// n = (t * H + h) * W + w.
void oracle_token_position(int64_t n, int T, int H, int W, int* pos) {
    (void)T;
    pos[0] = static_cast<int>(n / (static_cast<int64_t>(H) * W));
    pos[1] = static_cast<int>((n / W) % H);
    pos[2] = static_cast<int>(n % W);
}

// Fused prologue over one [B, N, heads, d] bf16 tensor: RMSNorm over each
// head's d channels with gains gamma[d], then 3D RoPE at the token's grid
// position.  Output is fp64 in the same layout.  Returns 0, or -1 on bad sizes.
int oracle_qk_norm_rope(const uint16_t* x, int B, int64_t N, int heads, int d,
                        const float* gamma, int T, int H, int W, double theta,
                        double eps, double* out, int nthreads) {
    if (B < 0 || N < 0 || heads <= 0 || d <= 0 || d % 6 != 0) return -1;
    if (static_cast<int64_t>(T) * H * W != N) return -1;
    std::vector<double> g(d);
    for (int i = 0; i < d; ++i) g[i] = static_cast<double>(gamma[i]);
    parallel_for(static_cast<int64_t>(B) * N, nthreads, [&](int64_t bn) {
        int b = static_cast<int>(bn / (N > 0 ? N : 1));
        int64_t n = bn % (N > 0 ? N : 1);
        int pos[3];
        oracle_token_position(n, T, H, W, pos);
        std::vector<double> xv(d), yv(d);
        for (int h = 0; h < heads; ++h) {
            for (int c = 0; c < d; ++c) xv[c] = bf16_to_double(x[bshd_index(b, n, h, c, N, heads, d)]);
            oracle_rmsnorm(xv.data(), d, g.data(), eps, yv.data());
            oracle_rope3d(yv.data(), d, pos, theta);
            for (int c = 0; c < d; ++c) out[bshd_index(b, n, h, c, N, heads, d)] = yv[c];
        }
    });
    return 0;
}

// Same as oracle_qk_norm_rope for a list of flattened tokens tok[i] = b*N + n
// only; out layout [ntok, heads, d], fp64.
int oracle_qk_norm_rope_tokens(const uint16_t* x, int B, int64_t N, int heads, int d, const float* gamma,
                               int T, int H, int W, double theta, double eps, const int64_t* tok,
                               int64_t ntok, double* out, int nthreads) {
    if (B < 0 || N < 0 || heads <= 0 || d <= 0 || d % 6 != 0) return -1;
    if (static_cast<int64_t>(T) * H * W != N) return -1;
    std::vector<double> g(d);
    for (int i = 0; i < d; ++i) g[i] = static_cast<double>(gamma[i]);
    parallel_for(ntok, nthreads, [&](int64_t i) {
        int b = static_cast<int>(tok[i] / N);
        int64_t n = tok[i] % N;
        int pos[3];
        oracle_token_position(n, T, H, W, pos);
        std::vector<double> xv(d), yv(d);
        for (int h = 0; h < heads; ++h) {
            for (int c = 0; c < d; ++c) xv[c] = bf16_to_double(x[bshd_index(b, n, h, c, N, heads, d)]);
            oracle_rmsnorm(xv.data(), d, g.data(), eps, yv.data());
            oracle_rope3d(yv.data(), d, pos, theta);
            for (int c = 0; c < d; ++c) out[(i * heads + h) * d + c] = yv[c];
        }
    });
    return 0;
}

// Round doubles to bf16 bit patterns, nearest-even.
void oracle_round_bf16(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16_rne(x[i]);
}

// The fused prologue with its single rounding to bf16 applied, for whole
// tensors too large to hold in fp64: out is bf16 bits, layout of x.
int oracle_qk_norm_rope_bf16(const uint16_t* x, int B, int64_t N, int heads, int d, const float* gamma,
                             int T, int H, int W, double theta, double eps, uint16_t* out, int nthreads) {
    if (B < 0 || N < 0 || heads <= 0 || d <= 0 || d % 6 != 0) return -1;
    if (static_cast<int64_t>(T) * H * W != N) return -1;
    std::vector<double> g(d);
    for (int i = 0; i < d; ++i) g[i] = static_cast<double>(gamma[i]);
    parallel_for(static_cast<int64_t>(B) * N, nthreads, [&](int64_t bn) {
        int b = static_cast<int>(bn / N);
        int64_t n = bn % N;
        int pos[3];
        oracle_token_position(n, T, H, W, pos);
        std::vector<double> xv(d), yv(d);
        for (int h = 0; h < heads; ++h) {
            for (int c = 0; c < d; ++c) xv[c] = bf16_to_double(x[bshd_index(b, n, h, c, N, heads, d)]);
            oracle_rmsnorm(xv.data(), d, g.data(), eps, yv.data());
            oracle_rope3d(yv.data(), d, pos, theta);
            for (int c = 0; c < d; ++c) out[bshd_index(b, n, h, c, N, heads, d)] = double_to_bf16_rne(yv[c]);
        }
    });
    return 0;
}

// Number of blocks covering N tokens (the last one may be partial).
int64_t oracle_num_blocks(int64_t N, int block) { return (N + block - 1) / block; }

// KV blocks kept per query block: the top (1 - sparsity) fraction of nkv,
// rounded up, at least 1 (a tiny slack absorbs binary rounding of exact
// products such as 0.25 * 4).
int64_t oracle_k_blocks(int64_t nkv, double sparsity) {
    double want = std::ceil((1.0 - sparsity) * static_cast<double>(nkv) - 1e-9);
    int64_t k = static_cast<int64_t>(want);
    if (k < 1) k = 1;
    if (k > nkv) k = nkv;
    return k;
}

// Router step 1, block pooling: the mean of each block's tokens, per (b, h),
// accumulated in fp64 in token order, divided by the block's real length
// (the tail block is shorter), then rounded to fp32.
// pooled layout: [B, heads, nblk, d].
int oracle_pool(const uint16_t* x, int B, int64_t N, int heads, int d, int block,
                float* pooled, int nthreads) {
    if (block <= 0 || d <= 0 || heads <= 0) return -1;
    const int64_t nblk = oracle_num_blocks(N, block);
    parallel_for(static_cast<int64_t>(B) * heads, nthreads, [&](int64_t bh) {
        int b = static_cast<int>(bh / heads), h = static_cast<int>(bh % heads);
        std::vector<double> acc(d);
        for (int64_t i = 0; i < nblk; ++i) {
            int64_t n0 = i * block, n1 = std::min<int64_t>(N, n0 + block);
            std::fill(acc.begin(), acc.end(), 0.0);
            for (int64_t n = n0; n < n1; ++n)
                for (int c = 0; c < d; ++c) acc[c] += bf16_to_double(x[bshd_index(b, n, h, c, N, heads, d)]);
            double len = static_cast<double>(n1 - n0);
            for (int c = 0; c < d; ++c)
                pooled[(bh * nblk + i) * d + c] = static_cast<float>(acc[c] / len);
        }
    });
    return 0;
}

// Router step 2, block scores: S[i, j] = (qbar_i . kbar_j) / sqrt(d), the dot
// product taken in fp64 over the fp32 pooled vectors, then rounded to fp32.
// scores layout: [B * heads, nblk, nblk].
int oracle_block_scores(const float* qp, const float* kp, int64_t BH, int64_t nblk, int d,
                        float* scores, int nthreads) {
    const double inv_sqrt_d = 1.0 / std::sqrt(static_cast<double>(d));
    parallel_for(BH * nblk, nthreads, [&](int64_t bhi) {
        int64_t bh = bhi / nblk;
        const float* qi = qp + bhi * d;
        for (int64_t j = 0; j < nblk; ++j) {
            const float* kj = kp + (bh * nblk + j) * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += static_cast<double>(qi[c]) * static_cast<double>(kj[c]);
            scores[bhi * nblk + j] = static_cast<float>(dot * inv_sqrt_d);
        }
    });
    return 0;
}

// Router step 3, selection: for each row of `scores` keep the k highest
// entries, ties going to the lower block index, and emit the kept indices in
// ascending order.  idx layout: [rows, k].
int oracle_topk(const float* scores, int64_t rows, int64_t ncols, int64_t k, int32_t* idx,
                int nthreads) {
    if (k < 1 || k > ncols) return -1;
    parallel_for(rows, nthreads, [&](int64_t r) {
        const float* s = scores + r * ncols;
        std::vector<int32_t> order(ncols);
        for (int64_t j = 0; j < ncols; ++j) order[j] = static_cast<int32_t>(j);
        std::sort(order.begin(), order.end(), [s](int32_t a, int32_t b) {
            if (s[a] != s[b]) return s[a] > s[b];
            return a < b;
        });
        std::vector<int32_t> kept(order.begin(), order.begin() + k);
        std::sort(kept.begin(), kept.end());
        for (int64_t i = 0; i < k; ++i) idx[r * k + i] = kept[i];
    });
    return 0;
}

// The whole router: pool Q and K, score, select.  Writes idx [B, heads, nblk, k]
// and, if scores_out is not null, the fp32 scores [B, heads, nblk, nblk].
// Returns k, or -1 on bad arguments.
int64_t oracle_route(const uint16_t* q, const uint16_t* k, int B, int64_t N, int heads, int d,
                     double sparsity, int block, int32_t* idx, float* scores_out, int nthreads) {
    if (B <= 0 || N <= 0 || heads <= 0 || d <= 0 || block <= 0) return -1;
    if (!(sparsity >= 0.0 && sparsity < 1.0)) return -1;
    const int64_t nblk = oracle_num_blocks(N, block);
    const int64_t kk = oracle_k_blocks(nblk, sparsity);
    const int64_t BH = static_cast<int64_t>(B) * heads;
    std::vector<float> qp(BH * nblk * d), kp(BH * nblk * d);
    oracle_pool(q, B, N, heads, d, block, qp.data(), nthreads);
    oracle_pool(k, B, N, heads, d, block, kp.data(), nthreads);
    std::vector<float> sc_local;
    float* sc = scores_out;
    if (sc == nullptr) {
        sc_local.resize(BH * nblk * nblk);
        sc = sc_local.data();
    }
    oracle_block_scores(qp.data(), kp.data(), BH, nblk, d, sc, nthreads);
    oracle_topk(sc, BH * nblk, nblk, kk, idx, nthreads);
    return kk;
}

// Attention output of selected query rows, fp64.  Row r = rows[i] encodes
// (b, h, n) as r = (b * heads + h) * N + n.  For each row:
//   logits l_j = scale * (q_n . k_j) over the row's key set,
//   o = sum_j exp(l_j - max l) v_j / sum_j exp(l_j - max l).
// Key set: every token (dense, block_idx == null) or the tokens of the KV
// blocks listed for the row's query block n / block (block_idx layout
// [B, heads, nblk, kblocks]).  No causal mask (bidirectional attention).
// out layout: [nrows, d].
int oracle_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B,
                          int64_t N, int heads, int d, const int32_t* block_idx,
                          int64_t kblocks, int block, double scale, const int64_t* rows,
                          int64_t nrows, double* out, int nthreads) {
    if (B <= 0 || N <= 0 || heads <= 0 || d <= 0) return -1;
    const int64_t nblk = oracle_num_blocks(N, block > 0 ? block : 1);
    parallel_for(nrows, nthreads, [&](int64_t i) {
        const int64_t r = rows[i];
        const int64_t bh = r / N;
        const int64_t n = r % N;
        const int b = static_cast<int>(bh / heads), h = static_cast<int>(bh % heads);
        std::vector<double> qv(d);
        for (int c = 0; c < d; ++c) qv[c] = bf16_to_double(q[bshd_index(b, n, h, c, N, heads, d)]);
        // the key set
        std::vector<int64_t> keys;
        if (block_idx == nullptr) {
            keys.resize(N);
            for (int64_t j = 0; j < N; ++j) keys[j] = j;
        } else {
            const int32_t* list = block_idx + ((bh * nblk) + n / block) * kblocks;
            for (int64_t t = 0; t < kblocks; ++t) {
                int64_t j0 = static_cast<int64_t>(list[t]) * block;
                int64_t j1 = std::min<int64_t>(N, j0 + block);
                for (int64_t j = j0; j < j1; ++j) keys.push_back(j);
            }
        }
        std::vector<double> logit(keys.size());
        double m = -INFINITY;
        for (size_t t = 0; t < keys.size(); ++t) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += qv[c] * bf16_to_double(k[bshd_index(b, keys[t], h, c, N, heads, d)]);
            logit[t] = scale * dot;
            if (logit[t] > m) m = logit[t];
        }
        std::vector<double> acc(d, 0.0);
        double denom = 0.0;
        for (size_t t = 0; t < keys.size(); ++t) {
            double p = std::exp(logit[t] - m);
            denom += p;
            for (int c = 0; c < d; ++c) acc[c] += p * bf16_to_double(v[bshd_index(b, keys[t], h, c, N, heads, d)]);
        }
        for (int c = 0; c < d; ++c) out[i * d + c] = acc[c] / denom;
    });
    return 0;
}

// The prologue with the RMSNorm spanning the token's whole hidden state (all
// heads, heads * d channels, one gain per hidden channel) instead of each
// head: the other reading of "QK-RMSNorm" in the cocoloop page's fused-operator
// paragraph.  Then the same per-head 3D RoPE, and one rounding to bf16:
//   r = 1 / sqrt(sum over all heads and channels of x^2 / (heads * d) + eps)
//   y[h, c] = RoPE_h(x[h, :] * r * gamma[h * d + :])[c]
// gamma: fp32 [heads * d].  out: bf16 bits, layout of x.
int oracle_qk_fullnorm_rope_bf16(const uint16_t* x, int B, int64_t N, int heads, int d, const float* gamma,
                                 int T, int H, int W, double theta, double eps, uint16_t* out, int nthreads) {
    if (B < 0 || N < 0 || heads <= 0 || d <= 0 || d % 6 != 0) return -1;
    if (static_cast<int64_t>(T) * H * W != N) return -1;
    parallel_for(static_cast<int64_t>(B) * N, nthreads, [&](int64_t bn) {
        const int b = static_cast<int>(bn / N);
        const int64_t n = bn % N;
        int pos[3];
        oracle_token_position(n, T, H, W, pos);
        double ss = 0.0;
        for (int h = 0; h < heads; ++h)
            for (int c = 0; c < d; ++c) {
                const double v = bf16_to_double(x[bshd_index(b, n, h, c, N, heads, d)]);
                ss += v * v;
            }
        const double r = 1.0 / std::sqrt(ss / (static_cast<double>(heads) * d) + eps);
        std::vector<double> yv(d);
        for (int h = 0; h < heads; ++h) {
            for (int c = 0; c < d; ++c)
                yv[c] = bf16_to_double(x[bshd_index(b, n, h, c, N, heads, d)]) * r *
                        static_cast<double>(gamma[h * d + c]);
            oracle_rope3d(yv.data(), d, pos, theta);
            for (int c = 0; c < d; ++c) out[bshd_index(b, n, h, c, N, heads, d)] = double_to_bf16_rne(yv[c]);
        }
    });
    return 0;
}

// Gated residual followed by the AdaLN update, per token row of width C
// (cocoloop page, fused-operator paragraph: the AdaLN update and the gated
// residual path; definitions as in DiT blocks).  For batch b and row r:
//   h = x + gate[b] * f                 (f == NULL: h = x, the AdaLN update alone)
//   h is rounded once to bf16 (that is the tensor the block passes on)
//   mu = mean(h), var = mean((h - mu)^2) over the C channels of the rounded h
//   y = (h - mu) / sqrt(var + eps) * (1 + scale[b]) + shift[b]
// x, f: bf16 [B, R, C]; gate, shift, scale: fp32 [B, C].  h_bits receives
// the rounded h (bf16 bits), y the fp64 result before its rounding.
int oracle_residual_adaln(const uint16_t* x, const uint16_t* f, const float* gate, const float* shift,
                          const float* scale, int B, int64_t R, int C, double eps, uint16_t* h_bits, double* y,
                          int nthreads) {
    if (B < 1 || R < 0 || C < 1 || eps < 0) return 1;
    parallel_for(static_cast<int64_t>(B) * R, nthreads, [&](int64_t br) {
        const int b = static_cast<int>(br / R);
        const int64_t base = br * C;
        std::vector<double> h(C);
        for (int c = 0; c < C; ++c) {
            double v = bf16_to_double(x[base + c]);
            if (f) v += static_cast<double>(gate[static_cast<int64_t>(b) * C + c]) * bf16_to_double(f[base + c]);
            h_bits[base + c] = double_to_bf16_rne(v);
            h[c] = bf16_to_double(h_bits[base + c]);
        }
        double mu = 0.0;
        for (int c = 0; c < C; ++c) mu += h[c];
        mu /= C;
        double var = 0.0;
        for (int c = 0; c < C; ++c) var += (h[c] - mu) * (h[c] - mu);
        var /= C;
        const double rstd = 1.0 / std::sqrt(var + eps);
        for (int c = 0; c < C; ++c) {
            const int64_t bc = static_cast<int64_t>(b) * C + c;
            y[base + c] = (h[c] - mu) * rstd * (1.0 + static_cast<double>(scale[bc])) + static_cast<double>(shift[bc]);
        }
    });
    return 0;
}

// SwiGLU activation (cocoloop page, fused-operator paragraph): for each row of
// a bf16 [R, 2F] tensor whose halves are a = [0, F) and b = [F, 2F),
// out = silu(a) * b = a / (1 + exp(-a)) * b, in fp64.
int oracle_swiglu(const uint16_t* in, int64_t R, int F, double* out, int nthreads) {
    if (R < 0 || F < 1) return 1;
    parallel_for(R, nthreads, [&](int64_t r) {
        for (int i = 0; i < F; ++i) {
            const double a = bf16_to_double(in[r * 2 * F + i]);
            const double bv = bf16_to_double(in[r * 2 * F + F + i]);
            out[r * F + i] = a / (1.0 + std::exp(-a)) * bv;
        }
    });
    return 0;
}

// Cache-DiT reuse decision quantity (cocoloop page, Cache-DiT paragraph: a
// residual-difference threshold of 0.04 / 0.08 decides reuse between
// adjacent denoising steps): the relative L1 difference of the current
// step's residual to the previous step's,
//   rel = sum_i |cur_i - prev_i| / sum_i |prev_i|   (fp64; +inf if prev is 0
//   everywhere and cur is not, 0 if both are),
// over n bf16 values.  Reuse when rel < threshold.
double oracle_residual_diff(const uint16_t* cur, const uint16_t* prev, int64_t n) {
    double num = 0.0, den = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        const double a = bf16_to_double(cur[i]), b = bf16_to_double(prev[i]);
        num += std::fabs(a - b);
        den += std::fabs(b);
    }
    if (den == 0.0) return num == 0.0 ? 0.0 : INFINITY;
    return num / den;
}

}  // extern "C"
