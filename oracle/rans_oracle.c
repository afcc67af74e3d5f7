/*
 * Oracle rANS coder for the DCKV codec -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain scalar C, written for readability, not speed.  Only the test-suite, the
 * smoke check and the CPU-baseline leg of the benchmark load this file's library.
 *
 * Source: "DCKV: Learned Transform Coding of the Prompt KV Cache in Hybrid Language
 * Models" (trove.briskstack.com summary), section "How it works", bullet "Coding":
 * codes are rANS-coded under Laplace distributions.  The coder parameters below are
 * the ones the codec specification fixes: 32 interleaved 32-bit states per chunk,
 * 16-bit renormalisation words, 16-bit frequency precision.
 *
 * Definitions (M = 2^16 total frequency, L = 2^16 lower state bound):
 *   symbol i of a chunk (i = 0..S-1) is coded by state (i mod 32);
 *   encoder: every state starts at L; symbols are visited from i = S-1 down to 0;
 *            before coding a symbol of frequency f, while x >= f * 2^16 the low 16 bits
 *            of x are emitted and x >>= 16; then x = (x / f) * M + (x mod f) + cdf;
 *   stream:  the 32 final states, then the emitted words in reverse emission order
 *            (that is, in the order the decoder consumes them);
 *   decoder: symbols i = 0..S-1: slot = x mod M, the symbol s with
 *            cdf[s] <= slot < cdf[s+1], x = f * (x >> 16) + slot - cdf[s], and if
 *            x < L then x = (x << 16) | next word.
 */
#include <stdint.h>
#include <stddef.h>

#define ORACLE_LANES 32
#define ORACLE_L 65536u
#define ORACLE_ALPHABET 510

/* Encode S symbols.  sym[i] in [0,510), scl[i] in [0,64) selects the table row.
 * freq: [64][510], cdf: [64][511].  Writes 32 states and the words (decoder order).
 * Returns the number of words, or -1 if words_cap is too small or a symbol is invalid. */
long oracle_rans_encode(const uint16_t *sym, const uint8_t *scl, long S,
                        const uint32_t *freq, const uint32_t *cdf,
                        uint32_t *states_out, uint16_t *words_out, long words_cap)
{
    uint32_t x[ORACLE_LANES];
    long n = 0;
    for (int j = 0; j < ORACLE_LANES; ++j) x[j] = ORACLE_L;
    /* emit into the tail of words_out, then move to the front */
    long pos = words_cap;
    for (long i = S - 1; i >= 0; --i) {
        int lane = (int)(i % ORACLE_LANES);
        int s = scl[i];
        int k = sym[i];
        if (s < 0 || s >= 64 || k < 0 || k >= ORACLE_ALPHABET) return -1;
        uint32_t f = freq[s * ORACLE_ALPHABET + k];
        uint32_t c = cdf[s * (ORACLE_ALPHABET + 1) + k];
        if (f == 0) return -1;
        uint64_t xs = x[lane];
        if (xs >= ((uint64_t)f << 16)) {
            if (pos == 0) return -1;
            words_out[--pos] = (uint16_t)(xs & 0xFFFFu);
            xs >>= 16;
            ++n;
        }
        xs = (xs / f) * 65536u + (xs % f) + c;
        x[lane] = (uint32_t)xs;
    }
    for (long w = 0; w < n; ++w) words_out[w] = words_out[pos + w];
    for (int j = 0; j < ORACLE_LANES; ++j) states_out[j] = x[j];
    return n;
}

/* Decode S symbols.  Returns the number of words consumed, -1 on a stream overrun,
 * -2 if a state leaves its range; sym_out receives the symbols. */
long oracle_rans_decode(const uint32_t *states_in, const uint16_t *words, long n_words,
                        const uint8_t *scl, long S, const uint32_t *freq, const uint32_t *cdf,
                        uint16_t *sym_out)
{
    uint32_t x[ORACLE_LANES];
    long w = 0;
    for (int j = 0; j < ORACLE_LANES; ++j) x[j] = states_in[j];
    for (long i = 0; i < S; ++i) {
        int lane = (int)(i % ORACLE_LANES);
        int s = scl[i];
        const uint32_t *cd = cdf + s * (ORACLE_ALPHABET + 1);
        const uint32_t *fr = freq + s * ORACLE_ALPHABET;
        uint32_t xs = x[lane];
        if (xs < ORACLE_L) return -2;
        uint32_t slot = xs & 0xFFFFu;
        /* binary search: largest k with cd[k] <= slot */
        int lo = 0, hi = ORACLE_ALPHABET; /* cd[lo] <= slot < cd[hi] */
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (cd[mid] <= slot) lo = mid; else hi = mid;
        }
        uint32_t f = fr[lo];
        uint64_t nx = (uint64_t)f * (xs >> 16) + slot - cd[lo];
        if (nx < ORACLE_L) {
            if (w >= n_words) return -1;
            nx = (nx << 16) | words[w++];
        }
        x[lane] = (uint32_t)nx;
        sym_out[i] = (uint16_t)lo;
    }
    return w;
}

/* Final decoder states (valid after a full decode: every state returns to L). */
int oracle_rans_states_after(const uint32_t *states_in, const uint16_t *words, long n_words,
                             const uint8_t *scl, long S, const uint32_t *freq,
                             const uint32_t *cdf, uint32_t *states_out)
{
    uint32_t x[ORACLE_LANES];
    long w = 0;
    for (int j = 0; j < ORACLE_LANES; ++j) x[j] = states_in[j];
    for (long i = 0; i < S; ++i) {
        int lane = (int)(i % ORACLE_LANES);
        int s = scl[i];
        const uint32_t *cd = cdf + s * (ORACLE_ALPHABET + 1);
        const uint32_t *fr = freq + s * ORACLE_ALPHABET;
        uint32_t xs = x[lane];
        uint32_t slot = xs & 0xFFFFu;
        int lo = 0, hi = ORACLE_ALPHABET;
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (cd[mid] <= slot) lo = mid; else hi = mid;
        }
        uint64_t nx = (uint64_t)fr[lo] * (xs >> 16) + slot - cd[lo];
        if (nx < ORACLE_L) {
            if (w >= n_words) return -1;
            nx = (nx << 16) | words[w++];
        }
        x[lane] = (uint32_t)nx;
    }
    for (int j = 0; j < ORACLE_LANES; ++j) states_out[j] = x[j];
    return 0;
}
