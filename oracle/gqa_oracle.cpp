// gqa_oracle.cpp -- TEST INFRASTRUCTURE, not part of the product.
//
// A plain, slow, obviously correct fp64 CPU oracle for single-token
// grouped-query attention (GQA) decode.  Only the test suite, the smoke check
// and the benchmark's CPU-baseline / reference arm may load it.  The CUDA
// library never links, loads or calls it, and the two share no code: no
// headers, no helpers, no constants.
//
// Sources, cited by page title and section:
//   [LLMS] "Grouped-Query Attention (GQA) and Multi-Query Attention (MQA):
//          Mathematical Foundations, Arithmetic Intensity, and KV-Cache
//          Scaling Mechanics" (llms.blog)
//   [AIT]  "Grouped-Query Attention Shares Keys Without Sharing Every Query"
//          (aitamer.news)
//
// What the oracle computes ([LLMS] section 2, "Grouped-Query Attention", the
// equation for Head_i and the group index g(i)):
//   R = H_Q / H_KV query heads per group, and query head h (0-based) reads
//   key/value head g = floor(h / R), the 0-based form of g(i) = floor((i-1)/R)+1.
//   For every batch row b and query head h:
//     s_t = scale * sum_i q[b,h,i] * K[b,t,g,i]          for t in [0, L_b)
//     w_t = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u)
//     out[b,h,:] = sum_t w_t * V[b,t,g,:]
//   All arithmetic is in double.  bf16 and f32 inputs convert to double
//   exactly, so the oracle sees exactly the values the GPU receives.
//
// Readings where the pages leave a step open (each also listed in the design
// notes):
//   * Decode step: the single query is the newest position, so the causal
//     mask M of [LLMS] section 2 keeps all L_b cached tokens (the current
//     token's key/value already appended) and drops positions t >= L_b.
//   * L_b = 0 gives out = 0 (the empty sum).
//   * d_k = d_v = D ([LLMS] section 2 sets d_k = d_v).
//   * scale is passed by the caller; [LLMS] section 2 uses 1/sqrt(d_k).
//
// Split-KV pieces (partial softmax state over a token range, and the
// log-sum-exp merge of partials) are written out as the plain definitions:
// for a token range T, lse_T = log sum_{t in T} exp(s_t) and
// o_T = sum_{t in T} exp(s_t - lse_T) v_t; merging ranges T_1..T_n gives
// out = sum_j exp(lse_j - LSE) o_j with LSE = log sum_j exp(lse_j).
//
// Multi-token step (prefill, or a chunk of a prompt after a cached prefix):
// sequence b brings n_b = cu_q[b+1] - cu_q[b] new query tokens whose keys and
// values are already the last n_b of its L_b cached tokens.  Its query token
// j (0-based) therefore sits at position p = L_b - n_b + j, and the causal
// mask M of [LLMS] section 2 (M[j][t] = 0 for t <= j, -inf after) becomes
// "key t is visible iff t <= p": the whole cached prefix plus the new tokens
// up to and including itself.  With no prefix (L_b = n_b) this is the s x s
// mask as written; with n_b = 1 it is the decode step above.  [LLMS]'s
// opening section names this prompt-processing phase (prefill) and says it
// is compute-bound; the arithmetic is the Head_i equation unchanged.
//
// Layouts (row-major, innermost last):
//   q   [B, H_Q, D]                  decode; [total_q, H_Q, D] multi-token,
//                                    rows cu_q[b] .. cu_q[b+1]-1 for sequence b
//   k,v [B, S_max, H_KV, D]      logical contiguous cache
//   out [n_pairs, D] in the order of `pairs`, or [B, H_Q, D] when pairs==NULL
//       (multi-token: [n_rows, D] for `rows`, or [total_q, H_Q, D])
//
// Build: g++ -O2 -std=c++17 -shared -fPIC -pthread gqa_oracle.cpp

#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

enum InputType { IN_BF16 = 0, IN_F32 = 1, IN_F64 = 2, IN_E4M3 = 3 };

// OCP 8-bit floating point, E4M3 encoding: sign bit 7, exponent bits 6..3 with
// bias 7, mantissa bits 2..0; exponent 0 is subnormal (m * 2^-9); S.1111.111 is
// NaN and there is no infinity, so the largest finite value is 448.
double decode_e4m3(uint8_t byte) {
    const int sign = byte >> 7, e = (byte >> 3) & 15, m = byte & 7;
    double mag;
    if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
    if (e == 0)
        mag = std::ldexp(static_cast<double>(m), -9);
    else
        mag = std::ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

// Exact widening of one stored element to double.
double load_elem(const void* base, int dtype, int64_t index) {
    if (dtype == IN_BF16) {
        uint16_t bits = static_cast<const uint16_t*>(base)[index];
        uint32_t wide = static_cast<uint32_t>(bits) << 16;  // bf16 is the top half of an f32
        float f;
        std::memcpy(&f, &wide, sizeof f);
        return static_cast<double>(f);
    }
    if (dtype == IN_F32) return static_cast<double>(static_cast<const float*>(base)[index]);
    if (dtype == IN_E4M3) return decode_e4m3(static_cast<const uint8_t*>(base)[index]);
    return static_cast<const double*>(base)[index];
}

struct Problem {
    const void* q;
    const void* k;
    const void* v;
    int q_dtype;
    int kv_dtype;
    const int32_t* seq_lens;
    int B, H_Q, H_KV, D;
    int64_t S_max;
    double scale;
    const double* k_scale = nullptr;  // [H_KV]: stored keys are multiplied by it (quantised caches)
    const double* v_scale = nullptr;  // [H_KV]: stored values likewise
};

int64_t q_index(const Problem& p, int b, int h, int i) {
    return (static_cast<int64_t>(b) * p.H_Q + h) * p.D + i;
}

int64_t kv_index(const Problem& p, int b, int64_t t, int g, int i) {
    return ((static_cast<int64_t>(b) * p.S_max + t) * p.H_KV + g) * p.D + i;
}

// Group index of query head h: [LLMS] section 2, g(i) = floor((i-1)/R) + 1,
// written 0-based.
int group_of(const Problem& p, int h) {
    int R = p.H_Q / p.H_KV;
    return h / R;
}

// Score s_t = scale * <q_h, k_t> for one token ([LLMS] section 2, the argument
// of the softmax in the Head_i equation).
double score(const Problem& p, int b, int h, int64_t t) {
    int g = group_of(p, h);
    double acc = 0.0;
    for (int i = 0; i < p.D; ++i)
        acc += load_elem(p.q, p.q_dtype, q_index(p, b, h, i)) *
               load_elem(p.k, p.kv_dtype, kv_index(p, b, t, g, i));
    const double ks = p.k_scale ? p.k_scale[g] : 1.0;
    return p.scale * ks * acc;
}

// Softmax weights over tokens [0, L_b), two passes: max, then exp and sum.
// Returns an empty vector when L_b == 0.
std::vector<double> softmax_weights(const Problem& p, int b, int h) {
    int64_t L = p.seq_lens[b];
    std::vector<double> s(static_cast<size_t>(L));
    double m = -std::numeric_limits<double>::infinity();
    for (int64_t t = 0; t < L; ++t) {
        s[t] = score(p, b, h, t);
        if (s[t] > m) m = s[t];
    }
    double sum = 0.0;
    for (int64_t t = 0; t < L; ++t) {
        s[t] = std::exp(s[t] - m);
        sum += s[t];
    }
    for (int64_t t = 0; t < L; ++t) s[t] /= sum;
    return s;
}

// out[b,h,:] = sum_t w_t * V[b,t,g,:]   ([LLMS] section 2, Head_i equation).
void attend_one(const Problem& p, int b, int h, double* out) {
    std::vector<double> w = softmax_weights(p, b, h);
    int g = group_of(p, h);
    const double vs = p.v_scale ? p.v_scale[g] : 1.0;
    for (int i = 0; i < p.D; ++i) out[i] = 0.0;
    for (int64_t t = 0; t < static_cast<int64_t>(w.size()); ++t)
        for (int i = 0; i < p.D; ++i)
            out[i] += w[t] * vs * load_elem(p.v, p.kv_dtype, kv_index(p, b, t, g, i));
}

int check_problem(const Problem& p) {
    if (!p.q || !p.k || !p.v || !p.seq_lens) return 1;
    if (p.B < 0 || p.H_Q <= 0 || p.H_KV <= 0 || p.D <= 0 || p.S_max < 0) return 1;
    if (p.H_Q % p.H_KV != 0) return 1;  // [LLMS] section 2: R = H_Q / G is a whole number
    if (p.q_dtype < IN_BF16 || p.q_dtype > IN_F64) return 1;
    if (p.kv_dtype < IN_BF16 || p.kv_dtype > IN_E4M3) return 1;
    for (int b = 0; b < p.B; ++b)
        if (p.seq_lens[b] < 0 || p.seq_lens[b] > p.S_max) return 1;
    return 0;
}

int thread_count(int requested, int64_t work) {
    int n = requested > 0 ? requested : static_cast<int>(std::thread::hardware_concurrency());
    if (n < 1) n = 1;
    if (work < n) n = static_cast<int>(work > 0 ? work : 1);
    return n;
}

}  // namespace

extern "C" {

// Full decode step, or a chosen list of (b, h) pairs.
//   pairs: NULL for all B*H_Q pairs (out is [B,H_Q,D]); else n_pairs rows of
//          (b, h) and out is [n_pairs, D].
//   n_threads <= 0 uses every hardware thread.
// Returns 0 on success, 1 on invalid arguments (nothing written).
int oracle_gqa_decode(const void* q, int q_dtype, const void* k, const void* v, int kv_dtype,
                      const int32_t* seq_lens, int B, int H_Q, int H_KV, int D, int64_t S_max,
                      double scale, const int32_t* pairs, int64_t n_pairs, double* out,
                      int n_threads) {
    Problem p{q, k, v, q_dtype, kv_dtype, seq_lens, B, H_Q, H_KV, D, S_max, scale};
    if (check_problem(p) || !out) return 1;
    int64_t n = pairs ? n_pairs : static_cast<int64_t>(B) * H_Q;
    if (n < 0) return 1;
    if (pairs) {
        for (int64_t j = 0; j < n; ++j)
            if (pairs[2 * j] < 0 || pairs[2 * j] >= B || pairs[2 * j + 1] < 0 ||
                pairs[2 * j + 1] >= H_Q)
                return 1;
    }
    int nt = thread_count(n_threads, n);
    std::vector<std::thread> pool;
    for (int w = 0; w < nt; ++w) {
        pool.emplace_back([&, w]() {
            for (int64_t j = w; j < n; j += nt) {
                int b = pairs ? pairs[2 * j] : static_cast<int>(j / H_Q);
                int h = pairs ? pairs[2 * j + 1] : static_cast<int>(j % H_Q);
                attend_one(p, b, h, out + j * D);
            }
        });
    }
    for (auto& t : pool) t.join();
    return 0;
}

// oracle_gqa_decode for a cache whose stored keys and values are multiplied by
// per-KV-head factors k_scale[g], v_scale[g] (e.g. an 8-bit cache with
// kv_dtype 3 = E4M3): K = stored_k * k_scale[g], V = stored_v * v_scale[g].
int oracle_gqa_decode_scaled(const void* q, int q_dtype, const void* k, const void* v, int kv_dtype,
                             const double* k_scale, const double* v_scale, const int32_t* seq_lens,
                             int B, int H_Q, int H_KV, int D, int64_t S_max, double scale,
                             const int32_t* pairs, int64_t n_pairs, double* out, int n_threads) {
    Problem p{q, k, v, q_dtype, kv_dtype, seq_lens, B, H_Q, H_KV, D, S_max, scale};
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    if (check_problem(p) || !out || !k_scale || !v_scale) return 1;
    int64_t n = pairs ? n_pairs : static_cast<int64_t>(B) * H_Q;
    if (n < 0) return 1;
    if (pairs) {
        for (int64_t j = 0; j < n; ++j)
            if (pairs[2 * j] < 0 || pairs[2 * j] >= B || pairs[2 * j + 1] < 0 ||
                pairs[2 * j + 1] >= H_Q)
                return 1;
    }
    int nt = thread_count(n_threads, n);
    std::vector<std::thread> pool;
    for (int w = 0; w < nt; ++w) {
        pool.emplace_back([&, w]() {
            for (int64_t j = w; j < n; j += nt) {
                int b = pairs ? pairs[2 * j] : static_cast<int>(j / H_Q);
                int h = pairs ? pairs[2 * j + 1] : static_cast<int>(j % H_Q);
                attend_one(p, b, h, out + j * D);
            }
        });
    }
    for (auto& t : pool) t.join();
    return 0;
}

// Decoded value of every E4M3 byte 0..255 (out[256]), for pinning the decoder.
void oracle_e4m3_table(double* out) {
    for (int i = 0; i < 256; ++i) out[i] = decode_e4m3(static_cast<uint8_t>(i));
}

// The normalised softmax weights w_t, t in [0, L_b), of one (b, h) pair.
// w must hold seq_lens[b] doubles.  Returns 0, or 1 on invalid arguments.
int oracle_attention_weights(const void* q, int q_dtype, const void* k, int kv_dtype,
                             const int32_t* seq_lens, int B, int H_Q, int H_KV, int D,
                             int64_t S_max, double scale, int b, int h, double* w) {
    Problem p{q, k, k, q_dtype, kv_dtype, seq_lens, B, H_Q, H_KV, D, S_max, scale};
    if (check_problem(p) || !w || b < 0 || b >= B || h < 0 || h >= H_Q) return 1;
    std::vector<double> ws = softmax_weights(p, b, h);
    for (size_t t = 0; t < ws.size(); ++t) w[t] = ws[t];
    return 0;
}

// Partial softmax state of one (b, h) pair over tokens [t0, t1) clipped to
// [0, L_b): lse = log sum_t exp(s_t) (natural log) and o = sum_t exp(s_t - lse) v_t.
// An empty range gives lse = -inf and o = 0.
int oracle_partial(const void* q, int q_dtype, const void* k, const void* v, int kv_dtype,
                   const int32_t* seq_lens, int B, int H_Q, int H_KV, int D, int64_t S_max,
                   double scale, int b, int h, int64_t t0, int64_t t1, double* lse, double* o) {
    Problem p{q, k, v, q_dtype, kv_dtype, seq_lens, B, H_Q, H_KV, D, S_max, scale};
    if (check_problem(p) || !lse || !o || b < 0 || b >= B || h < 0 || h >= H_Q) return 1;
    int64_t lo = t0 < 0 ? 0 : t0;
    int64_t hi = t1 > seq_lens[b] ? seq_lens[b] : t1;
    for (int i = 0; i < D; ++i) o[i] = 0.0;
    if (hi <= lo) {
        *lse = -std::numeric_limits<double>::infinity();
        return 0;
    }
    std::vector<double> s(static_cast<size_t>(hi - lo));
    double m = -std::numeric_limits<double>::infinity();
    for (int64_t t = lo; t < hi; ++t) {
        s[t - lo] = score(p, b, h, t);
        if (s[t - lo] > m) m = s[t - lo];
    }
    double sum = 0.0;
    for (int64_t t = lo; t < hi; ++t) sum += std::exp(s[t - lo] - m);
    double l = m + std::log(sum);
    int g = group_of(p, h);
    for (int64_t t = lo; t < hi; ++t) {
        double wt = std::exp(s[t - lo] - l);
        for (int i = 0; i < D; ++i) o[i] += wt * load_elem(p.v, p.kv_dtype, kv_index(p, b, t, g, i));
    }
    *lse = l;
    return 0;
}

// Log-sum-exp merge of n partials (lse[j], o[j*D .. j*D+D)) into out[D].
// All partials empty (every lse = -inf) gives out = 0.
int oracle_lse_combine(int64_t n, const double* lse, const double* o, int D, double* out) {
    if (n < 0 || D <= 0 || !out || (n > 0 && (!lse || !o))) return 1;
    double M = -std::numeric_limits<double>::infinity();
    for (int64_t j = 0; j < n; ++j)
        if (lse[j] > M) M = lse[j];
    for (int i = 0; i < D; ++i) out[i] = 0.0;
    if (n == 0 || M == -std::numeric_limits<double>::infinity()) return 0;
    double total = 0.0;
    for (int64_t j = 0; j < n; ++j) total += std::exp(lse[j] - M);
    for (int64_t j = 0; j < n; ++j) {
        double wj = std::exp(lse[j] - M) / total;
        for (int i = 0; i < D; ++i) out[i] += wj * o[j * D + i];
    }
    return 0;
}

// KV-cache size in bytes for one sequence-set: 2 (keys and values) x layers x
// tokens x KV heads x head dim x bytes per element.  [LLMS] section 1, "KV
// Cache Memory Footprint" (the Memory_KV formula with b*s tokens, 2-byte
// elements); [AIT], the cache-estimate paragraph (general bytes per element).
double oracle_kv_cache_bytes(int64_t layers, int64_t tokens, int64_t H_KV, int64_t d,
                             int64_t elem_bytes) {
    return 2.0 * static_cast<double>(layers) * static_cast<double>(tokens) *
           static_cast<double>(H_KV) * static_cast<double>(d) * static_cast<double>(elem_bytes);
}

// Rotary position embedding of every row of x [B, H, D] at position pos[b]
// ([LLMS] section 4, "Rotary Position Embeddings (RoPE) Interaction":
// R_{Theta,m} = diag(R_{theta_1,m}, ..., R_{theta_{d/2},m}), one 2x2 rotation
// by angle m * theta_i per coordinate pair).  Readings: theta_i =
// base^(-2(i-1)/d) for i = 1..d/2 (the RoFormer frequencies the page cites);
// pairing 0 rotates adjacent coordinates (2i, 2i+1), the block-diagonal form
// as written; pairing 1 rotates (i, i + d/2).  out is [B, H, D] double.
int oracle_rope(const void* x, int dtype, int B, int H, int D, const int32_t* pos, double base,
                int pairing, double* out) {
    if (!x || !pos || !out || B < 0 || H <= 0 || D <= 0 || D % 2 != 0 || !(base > 0.0)) return 1;
    if (dtype < IN_BF16 || dtype > IN_F64 || (pairing != 0 && pairing != 1)) return 1;
    const int half = D / 2;
    for (int b = 0; b < B; ++b) {
        const double m = static_cast<double>(pos[b]);
        for (int h = 0; h < H; ++h) {
            const int64_t row = (static_cast<int64_t>(b) * H + h) * D;
            for (int i = 0; i < half; ++i) {
                const double theta = std::pow(base, -2.0 * i / D);
                const double c = std::cos(m * theta), sn = std::sin(m * theta);
                const int i0 = pairing == 0 ? 2 * i : i;
                const int i1 = pairing == 0 ? 2 * i + 1 : i + half;
                const double x0 = load_elem(x, dtype, row + i0), x1 = load_elem(x, dtype, row + i1);
                out[row + i0] = x0 * c - x1 * sn;
                out[row + i1] = x0 * sn + x1 * c;
            }
        }
    }
    return 0;
}

// Multi-token causal attention (see the header comment): for every listed
// (query row i, query head h), with b the sequence whose span
// [cu_q[b], cu_q[b+1]) holds i, j = i - cu_q[b], n_b the span length and
// p = L_b - n_b + j:
//     s_t = scale * <q[i,h,:], K[b,t,g,:]>                 for t in [0, p]
//     out = sum_t softmax(s)_t * V[b,t,g,:]
// in double, two passes (max, then exp and sum), g = floor(h / R).
//   cu_q: [B+1], cu_q[0] = 0, non-decreasing, n_b <= L_b for every b.
//   rows: NULL for every row (out is [cu_q[B], H_Q, D]); else n_rows pairs
//         (i, h) and out is [n_rows, D].
// Returns 0, or 1 on invalid arguments (nothing written).
int oracle_gqa_prefill(const void* q, int q_dtype, const void* k, const void* v, int kv_dtype,
                       const int32_t* seq_lens, const int32_t* cu_q, int B, int H_Q, int H_KV, int D,
                       int64_t S_max, double scale, const int32_t* rows, int64_t n_rows, double* out,
                       int n_threads) {
    Problem p{q, k, v, q_dtype, kv_dtype, seq_lens, B, H_Q, H_KV, D, S_max, scale};
    if (check_problem(p) || !out || !cu_q || cu_q[0] != 0) return 1;
    for (int b = 0; b < B; ++b) {
        const int n_b = cu_q[b + 1] - cu_q[b];
        if (n_b < 0 || n_b > seq_lens[b]) return 1;
    }
    const int64_t total = cu_q[B];
    const int64_t n = rows ? n_rows : total * H_Q;
    if (n < 0) return 1;
    if (rows) {
        for (int64_t r = 0; r < n; ++r)
            if (rows[2 * r] < 0 || rows[2 * r] >= total || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= H_Q)
                return 1;
    }
    auto one = [&](int64_t i, int h, double* o) {
        int b = 0;
        while (cu_q[b + 1] <= i) ++b;  // the span holding row i (spans are non-empty here)
        const int64_t n_b = cu_q[b + 1] - cu_q[b];
        const int64_t pos = seq_lens[b] - n_b + (i - cu_q[b]);
        const int g = group_of(p, h);
        std::vector<double> s(static_cast<size_t>(pos + 1));
        double m = -std::numeric_limits<double>::infinity();
        for (int64_t t = 0; t <= pos; ++t) {
            double acc = 0.0;
            for (int e = 0; e < D; ++e)
                acc += load_elem(q, q_dtype, (i * H_Q + h) * D + e) * load_elem(k, kv_dtype, kv_index(p, b, t, g, e));
            s[t] = scale * acc;
            if (s[t] > m) m = s[t];
        }
        double sum = 0.0;
        for (int64_t t = 0; t <= pos; ++t) {
            s[t] = std::exp(s[t] - m);
            sum += s[t];
        }
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        for (int64_t t = 0; t <= pos; ++t)
            for (int e = 0; e < D; ++e) o[e] += (s[t] / sum) * load_elem(v, kv_dtype, kv_index(p, b, t, g, e));
    };
    int nt = thread_count(n_threads, n);
    std::vector<std::thread> pool;
    for (int w = 0; w < nt; ++w) {
        pool.emplace_back([&, w]() {
            for (int64_t r = w; r < n; r += nt) {
                const int64_t i = rows ? rows[2 * r] : r / H_Q;
                const int h = rows ? rows[2 * r + 1] : static_cast<int>(r % H_Q);
                one(i, h, out + r * D);
            }
        });
    }
    for (auto& t : pool) t.join();
    return 0;
}

int oracle_hardware_threads(void) {
    return static_cast<int>(std::thread::hardware_concurrency());
}

}  // extern "C"
