// Per-tag bit allocation of the token-mixed INT2/INT4 cache (host code): the per-tag
// distortion D_k(b) from calibration Q/K/V and the INT2/INT4 choice per tag under an
// average-bit budget ("TriAxialKV per-role mixed-precision KV quantization for agentic
// prefills", Facts: per-tag distortion, allocator, quantizer, leftover routing).
//
// D_k(b): every token of tag k quantized at b bits (the others exact), causal attention
// over the calibration prefill, output MSE per query head; max over heads, mean over
// requests, sum over layers.  The exact attention is computed once per query head and
// each (tag, b) only adds the change of its own tokens' terms.  b = 4: K and V per token, groups of 32 channels.  b = 2: K
// per channel over 32-token groups of the tag's tokens in order, V per token; the last
// < 32 tokens of the tag take the 4-bit per-token path for K and V.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

// One correctly rounded binary32 step each (the quantizer of the cache: fp32 scale from
// min and max, fp16 scale and zero, codes from the fp16 values widened back).
void quant_group(const float *x, int n, int stride, int bits, double *out) {
    float mn = x[0], mx = x[0];
    for (int i = 1; i < n; ++i) {
        mn = std::min(mn, x[i * stride]);
        mx = std::max(mx, x[i * stride]);
    }
    const float qmax = static_cast<float>((1 << bits) - 1);
    volatile float diff = mx - mn;   // each step rounded on its own
    volatile float s32 = diff / qmax;
    const float s = __half2float(__float2half_rn(s32));
    const float z = __half2float(__float2half_rn(mn));
    for (int i = 0; i < n; ++i) {
        int c = 0;
        if (s != 0.0f) {
            volatile float d = x[i * stride] - z;
            volatile float r = d / s;
            c = static_cast<int>(std::lrint(r));
            c = std::max(0, std::min(c, (1 << bits) - 1));
        }
        out[i * stride] = static_cast<double>(c) * static_cast<double>(s) + static_cast<double>(z);
    }
}

float bf16f(uint16_t b) {
    uint32_t u = static_cast<uint32_t>(b) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// K or V rows of the tag's tokens quantized in place (src exact floats, dst dequantized).
void quantize_tag(const float *kf, const float *vf, const std::vector<int> &toks, int D, int bits, double *kq,
                  double *vq) {
    const int n = static_cast<int>(toks.size());
    const int full = bits == 2 ? n / 32 * 32 : 0;   // tokens in complete 2-bit key groups
    std::vector<float> col(32);
    std::vector<double> res(32);
    for (int g = 0; g < full / 32; ++g)
        for (int d = 0; d < D; ++d) {
            for (int i = 0; i < 32; ++i) col[i] = kf[static_cast<long long>(toks[32 * g + i]) * D + d];
            quant_group(col.data(), 32, 1, 2, res.data());
            for (int i = 0; i < 32; ++i) kq[static_cast<long long>(toks[32 * g + i]) * D + d] = res[i];
        }
    for (int i = 0; i < n; ++i) {
        const long long t = toks[i];
        const int kb = i < full ? 0 : 4;   // 0: key already in a 2-bit group
        const int vb = i < full ? 2 : 4;
        for (int j = 0; j < D / 32; ++j) {
            if (kb) quant_group(kf + t * D + 32 * j, 32, 1, kb, kq + t * D + 32 * j);
            quant_group(vf + t * D + 32 * j, 32, 1, vb, vq + t * D + 32 * j);
        }
    }
}

}  // namespace

extern "C" {

int kvq_tag_distortion(int num_layers, int num_requests, int n_q_heads, int n_kv_heads, int head_dim, int T,
                       const uint16_t *Q, const uint16_t *K, const uint16_t *V, const int32_t *tags, int num_tags,
                       double *D2, double *D4, int64_t *counts) {
    if (num_layers < 1 || num_requests < 1 || n_q_heads < 1 || n_kv_heads < 1 || T < 1 || num_tags < 1)
        return kvq::host_fail(KVQ_EINVAL, "layers, requests, heads, T and num_tags must be positive");
    if (head_dim < 32 || head_dim % 32 || n_q_heads % n_kv_heads)
        return kvq::host_fail(KVQ_EINVAL, "head_dim must be a multiple of 32 and n_q_heads of n_kv_heads");
    if (!Q || !K || !V || !tags || !D2 || !D4 || !counts) return kvq::host_fail(KVQ_EINVAL, "null argument");
    const int D = head_dim, G = n_q_heads / n_kv_heads, R = num_requests, NL = num_layers;
    for (long long i = 0; i < static_cast<long long>(R) * T; ++i)
        if (tags[i] < 0 || tags[i] >= num_tags) return kvq::host_fail(KVQ_EINVAL, "tag out of range");
    // every worker holds a T x T fp64 score matrix and ~12 T x D rows: refuse sizes whose
    // buffers would not fit the 2 GB the workers share, before anything is allocated
    const double per_thread = 8.0 * (static_cast<double>(T) * T + 12.0 * static_cast<double>(T) * head_dim);
    if (per_thread > 2.0e9)
        return kvq::host_fail(KVQ_EINVAL, "T too large for the host calibration (worker buffers exceed 2 GB)");
    for (int k = 0; k < num_tags; ++k) counts[k] = 0;
    for (long long i = 0; i < static_cast<long long>(R) * T; ++i) ++counts[tags[i]];

    // Per (layer, request, kv head): the exact causal attention of each query head once
    // (scores s_ij, row max m_i, sum l_i, numerator N_i); quantizing tag k changes only
    // the terms j of tag k, so O'_i = (N_i + dN_i) / (l_i + dl_i) with dN, dl summed over
    // those terms (both weighted by exp(s - m_i) with the exact row max).
    // mse[((l * R + r) * num_tags + k) * 2 + bits_index][hq]: output MSE of query head hq.
    const long long TD = static_cast<long long>(T) * D;
    std::vector<double> mse(static_cast<size_t>(NL) * R * num_tags * 2 * n_q_heads, 0.0);
    std::vector<std::vector<int>> toks(static_cast<size_t>(R) * num_tags);
    for (int r = 0; r < R; ++r)
        for (int t = 0; t < T; ++t) toks[static_cast<size_t>(r) * num_tags + tags[static_cast<long long>(r) * T + t]].push_back(t);
    const long long ntask = static_cast<long long>(NL) * R * n_kv_heads;
    const double rs = 1.0 / std::sqrt(static_cast<double>(D));
    std::atomic<long long> next{0};
    std::atomic<int> failed{0};
    auto work_body = [&]() {
        std::vector<float> kf(TD), vf(TD);
        std::vector<double> kx(TD), vx(TD), kq(TD), vq(TD), qd(TD), S(static_cast<size_t>(T) * T), m(T), l(T),
            N(TD), dN(D), kxT(TD), kqT, sq;
        for (;;) {
            const long long task = next.fetch_add(1);
            if (task >= ntask) break;
            const int h = static_cast<int>(task % n_kv_heads);
            const int r = static_cast<int>((task / n_kv_heads) % R);
            const int lay = static_cast<int>(task / (static_cast<long long>(n_kv_heads) * R));
            const long long kvo = ((static_cast<long long>(lay) * R + r) * n_kv_heads + h) * TD;
            for (long long i = 0; i < TD; ++i) {
                kf[i] = bf16f(K[kvo + i]);
                vf[i] = bf16f(V[kvo + i]);
                kx[i] = kf[i];
                vx[i] = vf[i];
            }
            for (int j = 0; j < T; ++j)   // keys channel-major: score rows accumulate as axpys
                for (int c = 0; c < D; ++c) kxT[static_cast<long long>(c) * T + j] = kx[static_cast<long long>(j) * D + c];
            for (int gg = 0; gg < G; ++gg) {
                const int hq = h * G + gg;
                const long long qo = ((static_cast<long long>(lay) * R + r) * n_q_heads + hq) * TD;
                for (long long i = 0; i < TD; ++i) qd[i] = bf16f(Q[qo + i]);
                for (int i = 0; i < T; ++i) {
                    double *Si = S.data() + static_cast<size_t>(i) * T;
                    for (int j = 0; j <= i; ++j) Si[j] = 0.0;
                    for (int c = 0; c < D; ++c) {
                        const double qc = qd[static_cast<long long>(i) * D + c];
                        const double *kc = kxT.data() + static_cast<long long>(c) * T;
                        for (int j = 0; j <= i; ++j) Si[j] += qc * kc[j];
                    }
                    double mx = -INFINITY;
                    for (int j = 0; j <= i; ++j) {
                        Si[j] *= rs;
                        mx = std::max(mx, Si[j]);
                    }
                    m[i] = mx;
                    double li = 0.0;
                    double *Ni = N.data() + static_cast<long long>(i) * D;
                    for (int c = 0; c < D; ++c) Ni[c] = 0.0;
                    for (int j = 0; j <= i; ++j) {
                        const double pij = std::exp(Si[j] - mx);
                        Si[j] = pij;   // S now holds the exact weights exp(s_ij - m_i)
                        li += pij;
                        for (int c = 0; c < D; ++c) Ni[c] += pij * vx[j * D + c];
                    }
                    l[i] = li;
                }
                for (int k = 0; k < num_tags; ++k) {
                    const std::vector<int> &tk = toks[static_cast<size_t>(r) * num_tags + k];
                    if (tk.empty()) continue;
                    for (int bi = 0; bi < 2; ++bi) {
                        for (int t : tk)
                            for (int c = 0; c < D; ++c) {
                                kq[t * D + c] = kx[t * D + c];
                                vq[t * D + c] = vx[t * D + c];
                            }
                        quantize_tag(kf.data(), vf.data(), tk, D, bi == 0 ? 2 : 4, kq.data(), vq.data());
                        // the tag's quantized keys channel-major: a row's scores against its
                        // first cnt tag tokens accumulate as axpys over those tokens
                        const int nt = static_cast<int>(tk.size());
                        kqT.resize(static_cast<size_t>(D) * nt);
                        sq.resize(nt);
                        for (int ti = 0; ti < nt; ++ti)
                            for (int c = 0; c < D; ++c)
                                kqT[static_cast<size_t>(c) * nt + ti] = kq[static_cast<long long>(tk[ti]) * D + c];
                        double err = 0.0;
                        int cnt = 0;
                        for (int i = tk[0]; i < T; ++i) {
                            while (cnt < nt && tk[cnt] <= i) ++cnt;
                            for (int ti = 0; ti < cnt; ++ti) sq[ti] = 0.0;
                            for (int c = 0; c < D; ++c) {
                                const double qc = qd[static_cast<long long>(i) * D + c];
                                const double *kc = kqT.data() + static_cast<size_t>(c) * nt;
                                for (int ti = 0; ti < cnt; ++ti) sq[ti] += qc * kc[ti];
                            }
                            double dl = 0.0;
                            for (int c = 0; c < D; ++c) dN[c] = 0.0;
                            for (int ti = 0; ti < cnt; ++ti) {
                                const int t = tk[ti];
                                const double pq = std::exp(sq[ti] * rs - m[i]);
                                const double pe = S[static_cast<size_t>(i) * T + t];
                                dl += pq - pe;
                                for (int c = 0; c < D; ++c) dN[c] += pq * vq[t * D + c] - pe * vx[t * D + c];
                            }
                            const double *Ni = N.data() + static_cast<long long>(i) * D;
                            const double lq = l[i] + dl;
                            for (int c = 0; c < D; ++c) {
                                const double e = (Ni[c] + dN[c]) / lq - Ni[c] / l[i];
                                err += e * e;
                            }
                        }
                        mse[(((static_cast<size_t>(lay) * R + r) * num_tags + k) * 2 + bi) * n_q_heads + hq] =
                            err / static_cast<double>(TD);
                    }
                }
            }
        }
    };
    // a worker that cannot allocate its buffers stops the others and the call fails
    // (no exception leaves a worker thread)
    auto work = [&]() {
        try {
            work_body();
        } catch (...) {
            failed.store(1);
            next.store(ntask);
        }
    };
    // threads: the host's cores, at most 64, and as many as keep every worker's buffers
    // (the T x T fp64 scores and ~12 T x D rows) within about 2 GB
    const unsigned by_mem = static_cast<unsigned>(std::max(1.0, std::floor(2.0e9 / per_thread)));
    const unsigned nth = std::max(1u, std::min({std::thread::hardware_concurrency(), 64u, by_mem}));
    std::vector<std::thread> pool;
    for (unsigned i = 1; i < nth; ++i) pool.emplace_back(work);
    work();
    for (auto &th : pool) th.join();
    if (failed.load()) return kvq::host_fail(KVQ_EINVAL, "host memory exhausted during calibration");
    auto head_max = [&](int lay, int r, int k, int bi) {
        double w = 0.0;
        const double *e = mse.data() + (((static_cast<size_t>(lay) * R + r) * num_tags + k) * 2 + bi) * n_q_heads;
        for (int hq = 0; hq < n_q_heads; ++hq) w = std::max(w, e[hq]);
        return w;
    };
    for (int k = 0; k < num_tags; ++k) {
        double s2 = 0.0, s4 = 0.0;
        for (int l = 0; l < NL; ++l) {
            double m2 = 0.0, m4 = 0.0;
            for (int r = 0; r < R; ++r) {
                m2 += head_max(l, r, k, 0);
                m4 += head_max(l, r, k, 1);
            }
            s2 += m2 / R;
            s4 += m4 / R;
        }
        D2[k] = s2;
        D4[k] = s4;
    }
    return kvq::host_ok();
}

int kvq_tag_allocate(int num_tags, const double *D2, const double *D4, const int64_t *counts, double avg_bits,
                     int *bits, double *total_distortion) {
    if (num_tags < 1 || !D2 || !D4 || !counts || !bits) return kvq::host_fail(KVQ_EINVAL, "null argument or no tags");
    if (!(avg_bits >= 2.0 && avg_bits <= 4.0)) return kvq::host_fail(KVQ_EINVAL, "avg_bits must be in [2, 4]");
    std::vector<int> present;
    long long N = 0;
    for (int k = 0; k < num_tags; ++k) {
        if (counts[k] < 0) return kvq::host_fail(KVQ_EINVAL, "negative tag count");
        bits[k] = 4;
        if (counts[k] > 0) {
            present.push_back(k);
            N += counts[k];
        }
    }
    const double budget = avg_bits * static_cast<double>(N);   // total bits allowed
    const int P = static_cast<int>(present.size());
    if (P <= 22) {
        // exhaustive: bit i of the mask puts present tag i at INT2; the first mask of least
        // distortion in ascending order
        double best = INFINITY;
        uint32_t best_mask = 0;
        for (uint32_t mask = 0; mask < (1u << P); ++mask) {
            long long tb = 0;
            double dist = 0.0;
            for (int i = 0; i < P; ++i) {
                const int k = present[i];
                const bool two = (mask >> i) & 1u;
                tb += counts[k] * (two ? 2 : 4);
                dist += two ? D2[k] : D4[k];
            }
            if (static_cast<double>(tb) <= budget && dist < best) {
                best = dist;
                best_mask = mask;
            }
        }
        for (int i = 0; i < P; ++i) bits[present[i]] = ((best_mask >> i) & 1u) ? 2 : 4;
    } else {
        // greedy from all INT4: move to INT2 the tag with the least distortion added per
        // bit saved, (D2 - D4) / (2 n), until the budget holds (ties: lower tag index)
        long long tb = 4 * N;
        while (static_cast<double>(tb) > budget) {
            int pick = -1;
            double rate = INFINITY;
            for (int k : present) {
                if (bits[k] != 4) continue;
                const double r = (D2[k] - D4[k]) / (2.0 * static_cast<double>(counts[k]));
                if (r < rate) {
                    rate = r;
                    pick = k;
                }
            }
            if (pick < 0) break;
            bits[pick] = 2;
            tb -= 2 * counts[pick];
        }
    }
    if (total_distortion) {
        double dist = 0.0;
        for (int k : present) dist += bits[k] == 2 ? D2[k] : D4[k];
        *total_distortion = dist;
    }
    return kvq::host_ok();
}

}  // extern "C"
