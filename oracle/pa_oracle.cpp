// Paged-attention oracle — TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, single-threaded fp64 restatement of what the paged KV-cache
// path computes.  It exists to check the CUDA library; nothing in the product
// links, imports or calls it.  Only the tests, the smoke entry point and the
// benchmark's CPU-baseline leg may load it.  It shares no code, header, table
// or helper with the CUDA sources.
//
// Sources (page title, section):
//   [P1] "vLLM核心架构总览：PagedAttention、Continuous Batching、分布式推理等核心组件"
//        (5688vip.com, chapter 4), §4.1 PagedAttention: the KV cache is cut into
//        fixed-size physical blocks (16 or 32 tokens); logically contiguous KV
//        may be physically scattered; a block table keeps the mapping; prefix
//        blocks may be shared.
//   [P3] "从源码剖析 vLLM 的显存管理与连续批处理" (developer.cloud.tencent.cn),
//        §2.1 logical/physical block mapping (BlockTable.append_token: a new
//        physical block is taken when the logical block fills; physical address
//        = block address + offset), §2.2 one preallocated pool carved into equal
//        blocks, §2.3 attention receives block tables and gathers K/V by index
//        remapping before the matrix products.
//   [P4] "vLLM框架解析：PagedAttention技术如何实现LLM推理20倍加速"
//        (intelliparadigm.com), §2.3 zero-copy sharing of prefix blocks by
//        reference count, copy-on-write for isolation.
//   [P1] §4.2 preemption: a preempted sequence's KV blocks are swapped out to
//        CPU memory (or dropped and recomputed) and swapped back in later.
//   [P1] §4.3 chunked prefill: the prompt of a sequence is processed in chunks
//        that share the batch with decoding sequences.  Reading: a chunk is the
//        newest Q tokens of a sequence whose K/V (all L tokens, chunk included)
//        are already in the pool; chunk query i sits at position L - Q + i and
//        attends causally to the tokens at positions 0 .. L - Q + i.
//   [P4] §7 FP8 attention (the rest in FP16) as the next optimisation: here an
//        8-bit KV pool.  Readings (the pages fix no format): e4m3 codes (OCP
//        8-bit float, E4M3 "fn": 1 sign, 4 exponent bits with bias 7, 3
//        mantissa bits, no infinities, S.1111.111 = NaN, largest finite 448);
//        one fp32 scale per kv head for K and one for V; a stored value x
//        becomes code = e4m3(x / scale) with the division in fp32 (IEEE,
//        round to nearest) and the conversion rounding to nearest-even and
//        saturating to +-448; a code stands for e4m3_value(code) * scale.
//        Layout of the 8-bit pools (a reading as well; one (block, head) tile
//        of B*D bytes stays contiguous): K as [D/16][B][16] with the 16 dims
//        j of a vector at byte 4*((j%8)/2) + 2*(j/8) + j%2; V transposed, as
//        [D][B] with the tokens of each dim row in groups of 16 (8 when B=8)
//        and token u of a group of 16 at byte 4*((u%8)/2) + 2*(u/8) + u%2.
//
// Readings where the pages are silent (each is listed in the design notes):
//   * pool layout: an element (block b, kv head h, token t, dim d) lives at
//       (((b*Hkv + h)*(D/x) + d/x)*B + t)*x + d%x,   x = 16 / sizeof(elem)
//     i.e. each (block, head) tile is contiguous and is split along D into
//     16-byte vectors, vector index outer, token inner.
//   * slot encoding: slot = physical_block*B + offset; a negative slot is a
//     padding token and is skipped.
//   * GQA: query head h reads kv head h / (Hq/Hkv).
//   * context_lens[s] counts every token of sequence s, the newest included;
//     a sequence with no tokens yields an all-zero output.
//   * attention output: out[s,h,:] = sum_t softmax_t(scale * q.K_t) * V_t over
//     the logically ordered tokens t < context_lens[s]; all arithmetic in fp64
//     from the exact input values (fp16/bf16/fp32 widen exactly to fp64).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

namespace {

// Element type codes, defined here independently of the library's header.
constexpr int kF32 = 0;
constexpr int kF16 = 1;
constexpr int kBF16 = 2;

// Return codes.
constexpr int kOk = 0;
constexpr int kBadArg = 1;
constexpr int kBadBlockId = 2;
constexpr int kBadContextLen = 3;
constexpr int kBadSlot = 4;

int elem_size(int dtype) { return dtype == kF32 ? 4 : 2; }

bool dtype_ok(int dtype) { return dtype == kF32 || dtype == kF16 || dtype == kBF16; }

// IEEE binary32 bits -> double (exact).
double from_f32_bits(uint32_t bits) {
    float f;
    std::memcpy(&f, &bits, sizeof f);
    return static_cast<double>(f);
}

// bfloat16 is the top half of a binary32 -> exact.
double from_bf16_bits(uint16_t bits) { return from_f32_bits(static_cast<uint32_t>(bits) << 16); }

// IEEE binary16 -> double, decoded field by field (exact).
double from_f16_bits(uint16_t bits) {
    const int sign = bits >> 15;
    const int exponent = (bits >> 10) & 0x1f;
    const int mantissa = bits & 0x3ff;
    double v;
    if (exponent == 0) {
        v = std::ldexp(static_cast<double>(mantissa), -24);  // subnormal or zero
    } else if (exponent == 31) {
        v = mantissa ? std::numeric_limits<double>::quiet_NaN()
                     : std::numeric_limits<double>::infinity();
    } else {
        v = std::ldexp(static_cast<double>(mantissa + 1024), exponent - 25);
    }
    return sign ? -v : v;
}

// e4m3 bits -> double, field by field (exact).
double from_e4m3_bits(uint8_t bits) {
    const int sign = bits >> 7;
    const int exponent = (bits >> 3) & 0xf;
    const int mantissa = bits & 0x7;
    double v;
    if (exponent == 0xf && mantissa == 0x7) {
        v = std::numeric_limits<double>::quiet_NaN();
    } else if (exponent == 0) {
        v = std::ldexp(static_cast<double>(mantissa), -9);  // subnormal or zero: m * 2^-6 / 8
    } else {
        v = std::ldexp(static_cast<double>(mantissa + 8), exponent - 10);  // (1 + m/8) * 2^(e-7)
    }
    return sign ? -v : v;
}

// fp32 -> e4m3 bits: round to nearest, ties to even, at the precision of the
// binade of |v| (subnormal step 2^-9 below 2^-6), then saturate to 448.
uint8_t to_e4m3_bits(float v) {
    const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
    if (std::isnan(v)) return static_cast<uint8_t>(sign | 0x7f);
    const double a = std::fabs(static_cast<double>(v));
    if (a == 0.0) return sign;
    int e2 = 0;
    std::frexp(a, &e2);                        // a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1
    const int binade = std::max(e2 - 1, -6);   // normal binades start at 2^-6
    const double quantum = std::ldexp(1.0, binade - 3);
    double r = std::nearbyint(a / quantum) * quantum;  // default rounding mode: ties to even
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return sign;
    std::frexp(r, &e2);
    const int er = e2 - 1;
    if (er < -6) {
        return static_cast<uint8_t>(sign | static_cast<int>(std::ldexp(r, 9)));  // m * 2^-9
    }
    const int mant = static_cast<int>(std::ldexp(r, -er) * 8.0) - 8;
    return static_cast<uint8_t>(sign | ((er + 7) << 3) | mant);
}

// Element `index` of an array of `dtype`, widened to double.
double element(const void* base, int64_t index, int dtype) {
    if (dtype == kF32) {
        uint32_t b;
        std::memcpy(&b, static_cast<const uint8_t*>(base) + index * 4, 4);
        return from_f32_bits(b);
    }
    uint16_t b;
    std::memcpy(&b, static_cast<const uint8_t*>(base) + index * 2, 2);
    return dtype == kBF16 ? from_bf16_bits(b) : from_f16_bits(b);
}

// The byte order inside a 16-element group of the 8-bit pools: element j
// sits at 4*((j % 8) / 2) + 2*(j / 8) + j % 2.
int64_t e4m3_slot16(int64_t j) { return 4 * ((j % 8) / 2) + 2 * (j / 8) + j % 2; }

// Position of the code of (block, head, token, dim) in an 8-bit K pool.
int64_t e4m3_k_index(int64_t block, int64_t head, int64_t token, int64_t dim, int num_kv_heads, int block_size,
                     int head_dim) {
    const int64_t tile = block * num_kv_heads + head;
    const int64_t vector = tile * (head_dim / 16) + dim / 16;
    return (vector * block_size + token) * 16 + e4m3_slot16(dim % 16);
}

// Position of the code of (block, head, token, dim) in an 8-bit V pool.
int64_t e4m3_v_index(int64_t block, int64_t head, int64_t token, int64_t dim, int num_kv_heads, int block_size,
                     int head_dim) {
    const int64_t tile = block * num_kv_heads + head;
    const int64_t row = tile * head_dim + dim;
    const int64_t in_row = block_size == 8 ? token : 16 * (token / 16) + e4m3_slot16(token % 16);
    return row * block_size + in_row;
}

// Position of element (block, head, token, dim) in a pool array (see header).
int64_t pool_index(int64_t block, int64_t head, int64_t token, int64_t dim,
                   int num_kv_heads, int block_size, int head_dim, int vec) {
    const int64_t tile = block * num_kv_heads + head;
    const int64_t vector = tile * (head_dim / vec) + dim / vec;
    return (vector * block_size + token) * vec + dim % vec;
}

struct Shape {
    int block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks;
    int64_t num_blocks;
    int dtype;                       // queries (and K/V unless e4m3)
    const float* k_scale = nullptr;  // non-null: the pools hold e4m3 codes, one scale per kv head
    const float* v_scale = nullptr;
};

bool shape_ok(const Shape& s) {
    if (!dtype_ok(s.dtype)) return false;
    if (s.block_size <= 0 || s.num_seqs < 0 || s.num_q_heads <= 0 || s.num_kv_heads <= 0) return false;
    if (s.head_dim <= 0 || s.max_blocks < 0 || s.num_blocks <= 0) return false;
    if (s.num_q_heads % s.num_kv_heads != 0) return false;
    if ((s.k_scale == nullptr) != (s.v_scale == nullptr)) return false;
    if (s.k_scale && s.block_size != 8 && s.block_size % 16 != 0) return false;
    const int vec = s.k_scale ? 16 : 16 / elem_size(s.dtype);
    return s.head_dim % vec == 0;
}

// The logical K and V of one (sequence, kv head), gathered through the block
// table into contiguous fp64 arrays [L][D] in logical token order ([P3] §2.3).
int gather_sequence(const void* k_cache, const void* v_cache, const int32_t* table_row,
                    int context_len, int kv_head, const Shape& sh,
                    std::vector<double>& keys, std::vector<double>& values) {
    const bool e4m3 = sh.k_scale != nullptr;
    const int vec = e4m3 ? 16 : 16 / elem_size(sh.dtype);
    const int D = sh.head_dim;
    keys.assign(static_cast<size_t>(context_len) * D, 0.0);
    values.assign(static_cast<size_t>(context_len) * D, 0.0);
    for (int t = 0; t < context_len; ++t) {
        // Logical block t / B holds logical token t at offset t % B ([P3] §2.1).
        const int32_t physical = table_row[t / sh.block_size];
        if (physical < 0 || physical >= sh.num_blocks) return kBadBlockId;
        const int offset = t % sh.block_size;
        for (int d = 0; d < D; ++d) {
            const int64_t at = pool_index(physical, kv_head, offset, d, sh.num_kv_heads,
                                          sh.block_size, D, vec);
            if (e4m3) {  // a code stands for its e4m3 value times its kv head's scale
                const int64_t ka = e4m3_k_index(physical, kv_head, offset, d, sh.num_kv_heads, sh.block_size, D);
                const int64_t va = e4m3_v_index(physical, kv_head, offset, d, sh.num_kv_heads, sh.block_size, D);
                keys[static_cast<size_t>(t) * D + d] =
                    from_e4m3_bits(static_cast<const uint8_t*>(k_cache)[ka]) * static_cast<double>(sh.k_scale[kv_head]);
                values[static_cast<size_t>(t) * D + d] =
                    from_e4m3_bits(static_cast<const uint8_t*>(v_cache)[va]) * static_cast<double>(sh.v_scale[kv_head]);
            } else {
                keys[static_cast<size_t>(t) * D + d] = element(k_cache, at, sh.dtype);
                values[static_cast<size_t>(t) * D + d] = element(v_cache, at, sh.dtype);
            }
        }
    }
    return kOk;
}

// Scores z_t = scale * <q, K_t> for every logical token.
void scores_of(const double* q, const std::vector<double>& keys, int context_len, int D,
               double scale, std::vector<double>& z) {
    z.assign(context_len, 0.0);
    for (int t = 0; t < context_len; ++t) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * keys[static_cast<size_t>(t) * D + d];
        z[t] = scale * dot;
    }
}

int check_context_len(int len, const Shape& sh) {
    if (len < 0 || static_cast<int64_t>(len) > static_cast<int64_t>(sh.max_blocks) * sh.block_size)
        return kBadContextLen;
    return kOk;
}

// Attention of one query head of one sequence: two-pass softmax over all
// tokens, then the weighted sum of V.  `out` receives D doubles.
void attend_plain(const double* q, const std::vector<double>& keys,
                  const std::vector<double>& values, int context_len, int D, double scale,
                  double* out) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (context_len == 0) return;
    std::vector<double> z;
    scores_of(q, keys, context_len, D, scale, z);
    double zmax = z[0];
    for (int t = 1; t < context_len; ++t) zmax = std::fmax(zmax, z[t]);
    double denom = 0.0;
    std::vector<double> w(context_len);
    for (int t = 0; t < context_len; ++t) {
        w[t] = std::exp(z[t] - zmax);
        denom += w[t];
    }
    for (int t = 0; t < context_len; ++t) {
        const double p = w[t] / denom;
        for (int d = 0; d < D; ++d) out[d] += p * values[static_cast<size_t>(t) * D + d];
    }
}

// The same attention computed by token partitions of `part` tokens: each
// partition keeps its own max m_p, sum l_p = sum exp(z - m_p) and unnormalised
// accumulator a_p = sum exp(z - m_p) V; the partitions are then combined with
// weights exp(m_p - M), M = max_p m_p (the log-sum-exp merge).
void attend_partitioned(const double* q, const std::vector<double>& keys,
                        const std::vector<double>& values, int context_len, int D,
                        double scale, int part, double* out) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (context_len == 0) return;
    std::vector<double> z;
    scores_of(q, keys, context_len, D, scale, z);
    const int num_parts = (context_len + part - 1) / part;
    std::vector<double> m(num_parts), l(num_parts), acc(static_cast<size_t>(num_parts) * D, 0.0);
    for (int p = 0; p < num_parts; ++p) {
        const int t0 = p * part;
        const int t1 = std::min(context_len, t0 + part);
        double mp = z[t0];
        for (int t = t0 + 1; t < t1; ++t) mp = std::fmax(mp, z[t]);
        double lp = 0.0;
        for (int t = t0; t < t1; ++t) {
            const double e = std::exp(z[t] - mp);
            lp += e;
            for (int d = 0; d < D; ++d) acc[static_cast<size_t>(p) * D + d] += e * values[static_cast<size_t>(t) * D + d];
        }
        m[p] = mp;
        l[p] = lp;
    }
    double big = m[0];
    for (int p = 1; p < num_parts; ++p) big = std::fmax(big, m[p]);
    double denom = 0.0;
    for (int p = 0; p < num_parts; ++p) denom += std::exp(m[p] - big) * l[p];
    for (int p = 0; p < num_parts; ++p) {
        const double w = std::exp(m[p] - big) / denom;
        for (int d = 0; d < D; ++d) out[d] += w * acc[static_cast<size_t>(p) * D + d];
    }
}

int decode_common(double* out, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* block_tables, const int32_t* context_lens, float scale,
                  const Shape& sh, const int32_t* seq_ids, int num_selected, int partition) {
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return kBadArg;
    if (!shape_ok(sh)) return kBadArg;
    const int count = seq_ids ? num_selected : sh.num_seqs;
    const int group = sh.num_q_heads / sh.num_kv_heads;
    const int D = sh.head_dim;
    const double scale_d = static_cast<double>(scale);  // the fp32 scale, widened exactly
    std::vector<double> keys, values, qrow(D);
    for (int i = 0; i < count; ++i) {
        const int s = seq_ids ? seq_ids[i] : i;
        if (s < 0 || s >= sh.num_seqs) return kBadArg;
        const int len = context_lens[s];
        const int rc = check_context_len(len, sh);
        if (rc != kOk) return rc;
        const int32_t* row = block_tables + static_cast<int64_t>(s) * sh.max_blocks;
        for (int kvh = 0; kvh < sh.num_kv_heads; ++kvh) {
            const int g = gather_sequence(k_cache, v_cache, row, len, kvh, sh, keys, values);
            if (g != kOk) return g;
            for (int j = 0; j < group; ++j) {
                const int h = kvh * group + j;  // query head h reads kv head h / group
                for (int d = 0; d < D; ++d)
                    qrow[d] = element(q, (static_cast<int64_t>(s) * sh.num_q_heads + h) * D + d, sh.dtype);
                double* dst = out + (static_cast<int64_t>(i) * sh.num_q_heads + h) * D;
                if (partition > 0)
                    attend_partitioned(qrow.data(), keys, values, len, D, scale_d, partition, dst);
                else
                    attend_plain(qrow.data(), keys, values, len, D, scale_d, dst);
            }
        }
    }
    return kOk;
}

}  // namespace

extern "C" {

// Writes key/value rows [T][Hkv][D] into the pools through slot_mapping
// ([P3] §2.1 append_token: physical address = block address + offset).  A
// byte-for-byte element copy; slots < 0 are skipped.
int oracle_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int64_t num_blocks, int dtype) {
    if (!key || !value || !k_cache || !v_cache || (!slot_mapping && num_tokens > 0)) return kBadArg;
    if (!dtype_ok(dtype) || num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0)
        return kBadArg;
    const int es = elem_size(dtype);
    const int vec = 16 / es;
    if (head_dim % vec != 0) return kBadArg;
    for (int64_t i = 0; i < num_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        if (slot >= num_blocks * block_size) return kBadSlot;
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                const int64_t src = (i * num_kv_heads + h) * head_dim + d;
                const int64_t dst = pool_index(block, h, offset, d, num_kv_heads, block_size, head_dim, vec);
                std::memcpy(static_cast<uint8_t*>(k_cache) + dst * es,
                            static_cast<const uint8_t*>(key) + src * es, es);
                std::memcpy(static_cast<uint8_t*>(v_cache) + dst * es,
                            static_cast<const uint8_t*>(value) + src * es, es);
            }
        }
    }
    return kOk;
}

// Paged decode attention, fp64.  out: [num_selected or num_seqs][Hq][D]
// doubles.  seq_ids (optional) selects which sequences to compute, in order.
int oracle_decode(double* out, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* block_tables, const int32_t* context_lens, float scale,
                  int block_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                  int max_blocks_per_seq, int64_t num_blocks, int dtype, const int32_t* seq_ids,
                  int num_selected) {
    const Shape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim,
                   max_blocks_per_seq, num_blocks, dtype};
    return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh, seq_ids,
                         num_selected, 0);
}

// The same result reached through partitions of `partition_size` tokens and a
// log-sum-exp merge (the long-context split), fp64.
int oracle_decode_partitioned(double* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, const int32_t* context_lens, float scale,
                              int block_size, int num_seqs, int num_q_heads, int num_kv_heads,
                              int head_dim, int max_blocks_per_seq, int64_t num_blocks, int dtype,
                              const int32_t* seq_ids, int num_selected, int partition_size) {
    if (partition_size <= 0) return kBadArg;
    const Shape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim,
                   max_blocks_per_seq, num_blocks, dtype};
    return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh, seq_ids,
                         num_selected, partition_size);
}

// Paged prefill of query chunks ([P1] §4.3 chunked prefill): queries
// [T][Hq][D] with sequence s owning rows query_start[s] .. query_start[s+1]-1
// (Q_s of them, Q_s <= context_lens[s]); out [T][Hq][D] doubles.  Query i of
// sequence s attends to its first L_s - Q_s + i + 1 logical tokens.
int oracle_prefill(double* out, const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
                   float scale, int block_size, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                   int max_blocks_per_seq, int64_t num_blocks, int dtype) {
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start) return kBadArg;
    const Shape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, num_blocks, dtype};
    if (!shape_ok(sh)) return kBadArg;
    const int group = num_q_heads / num_kv_heads;
    const int D = head_dim;
    const double scale_d = static_cast<double>(scale);
    std::vector<double> keys, values, qrow(D);
    if (query_start[0] != 0) return kBadArg;
    for (int s = 0; s < num_seqs; ++s) {
        const int len = context_lens[s];
        const int rc = check_context_len(len, sh);
        if (rc != kOk) return rc;
        const int first = query_start[s];
        const int count = query_start[s + 1] - first;
        if (count < 0 || count > len) return kBadArg;
        const int32_t* row = block_tables + static_cast<int64_t>(s) * max_blocks_per_seq;
        for (int kvh = 0; kvh < num_kv_heads; ++kvh) {
            const int g = gather_sequence(k_cache, v_cache, row, len, kvh, sh, keys, values);
            if (g != kOk) return g;
            for (int i = 0; i < count; ++i) {
                const int visible = len - count + i + 1;  // positions 0 .. L - Q + i
                for (int j = 0; j < group; ++j) {
                    const int h = kvh * group + j;
                    const int64_t t = first + i;
                    for (int d = 0; d < D; ++d)
                        qrow[d] = element(q, (t * num_q_heads + h) * D + d, dtype);
                    attend_plain(qrow.data(), keys, values, visible, D, scale_d,
                                 out + (t * num_q_heads + h) * D);
                }
            }
        }
    }
    return kOk;
}

// Position of element (block, head, token, dim) in a pool of the given shape,
// exported so the layout itself can be pinned against hand-derived offsets.
// Copies whole physical blocks (every kv head, token and dimension of the K
// and of the V pool) from a source pool pair to a destination pool pair:
// block_mapping holds num_pairs (src, dst) block-id pairs.  The same pool as
// source and destination is the copy-on-write duplicate of a shared block
// ([P4] §2.3); a host-memory pool on one side is a swap-out or swap-in of a
// preempted sequence's blocks ([P1] §4.2).  Element by element through the
// pool layout, pairs in order.  A pair whose source id is negative is an empty
// entry and copies nothing (like a negative slot in the write); any other block
// id outside its pool is refused.
int oracle_copy_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                       const int64_t* block_mapping, int64_t num_pairs, int num_kv_heads,
                       int head_dim, int block_size, int64_t src_num_blocks,
                       int64_t dst_num_blocks, int dtype) {
    if (!dst_k || !dst_v || !src_k || !src_v || (!block_mapping && num_pairs > 0)) return kBadArg;
    if (!dtype_ok(dtype) || num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        src_num_blocks <= 0 || dst_num_blocks <= 0)
        return kBadArg;
    const int es = elem_size(dtype);
    const int vec = 16 / es;
    if (head_dim % vec != 0) return kBadArg;
    for (int64_t i = 0; i < num_pairs; ++i) {
        const int64_t src = block_mapping[2 * i];
        const int64_t dst = block_mapping[2 * i + 1];
        if (src < 0) continue;
        if (src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return kBadBlockId;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int t = 0; t < block_size; ++t) {
                for (int d = 0; d < head_dim; ++d) {
                    const int64_t from = pool_index(src, h, t, d, num_kv_heads, block_size, head_dim, vec);
                    const int64_t to = pool_index(dst, h, t, d, num_kv_heads, block_size, head_dim, vec);
                    std::memcpy(static_cast<uint8_t*>(dst_k) + to * es,
                                static_cast<const uint8_t*>(src_k) + from * es, es);
                    std::memcpy(static_cast<uint8_t*>(dst_v) + to * es,
                                static_cast<const uint8_t*>(src_v) + from * es, es);
                }
            }
        }
    }
    return kOk;
}

// The 8-bit pool's write: key/value rows [T][Hkv][D] (dtype) quantised to
// e4m3 codes with the kv head's scale and stored through slot_mapping like
// oracle_reshape_and_cache (pools of 1-byte elements, 16 per vector).
int oracle_reshape_and_cache_e4m3(const void* key, const void* value, void* k_cache, void* v_cache,
                                  const int64_t* slot_mapping, const float* k_scale, const float* v_scale,
                                  int64_t num_tokens, int num_kv_heads, int head_dim, int block_size,
                                  int64_t num_blocks, int dtype) {
    if (!key || !value || !k_cache || !v_cache || !k_scale || !v_scale || (!slot_mapping && num_tokens > 0))
        return kBadArg;
    if (!dtype_ok(dtype) || num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || head_dim % 16 != 0 || (block_size != 8 && block_size % 16 != 0))
        return kBadArg;
    for (int64_t i = 0; i < num_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        if (slot >= num_blocks * block_size) return kBadSlot;
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                const int64_t src = (i * num_kv_heads + h) * head_dim + d;
                const int64_t kdst = e4m3_k_index(block, h, offset, d, num_kv_heads, block_size, head_dim);
                const int64_t vdst = e4m3_v_index(block, h, offset, d, num_kv_heads, block_size, head_dim);
                const float kx = static_cast<float>(element(key, src, dtype));    // exact
                const float vx = static_cast<float>(element(value, src, dtype));
                static_cast<uint8_t*>(k_cache)[kdst] = to_e4m3_bits(kx / k_scale[h]);
                static_cast<uint8_t*>(v_cache)[vdst] = to_e4m3_bits(vx / v_scale[h]);
            }
        }
    }
    return kOk;
}

// Paged decode over e4m3 pools (queries and output in `dtype`), fp64; with
// partition > 0 the partitioned form with the log-sum-exp merge.
int oracle_decode_e4m3(double* out, const void* q, const void* k_cache, const void* v_cache,
                       const float* k_scale, const float* v_scale, const int32_t* block_tables,
                       const int32_t* context_lens, float scale, int block_size, int num_seqs,
                       int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                       int64_t num_blocks, int dtype, const int32_t* seq_ids, int num_selected,
                       int partition) {
    if (!k_scale || !v_scale || partition < 0) return kBadArg;
    Shape sh{block_size, num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, num_blocks, dtype};
    sh.k_scale = k_scale;
    sh.v_scale = v_scale;
    return decode_common(out, q, k_cache, v_cache, block_tables, context_lens, scale, sh, seq_ids,
                         num_selected, partition);
}

// The 8-bit pools' layout functions, for the pins.
int64_t oracle_e4m3_k_index(int64_t block, int head, int token, int dim, int num_kv_heads, int block_size,
                            int head_dim) {
    return e4m3_k_index(block, head, token, dim, num_kv_heads, block_size, head_dim);
}
int64_t oracle_e4m3_v_index(int64_t block, int head, int token, int dim, int num_kv_heads, int block_size,
                            int head_dim) {
    return e4m3_v_index(block, head, token, dim, num_kv_heads, block_size, head_dim);
}

// The format functions on their own, for the pins.
double oracle_e4m3_value(int bits) { return from_e4m3_bits(static_cast<uint8_t>(bits)); }
int oracle_e4m3_encode(float v) { return to_e4m3_bits(v); }

int64_t oracle_pool_index(int64_t block, int head, int token, int dim, int num_kv_heads,
                          int block_size, int head_dim, int dtype) {
    return pool_index(block, head, token, dim, num_kv_heads, block_size, head_dim,
                      16 / elem_size(dtype));
}

}  // extern "C"
