// policy.cu -- per-step policy: whether one attention call runs the sparse
// path or stays dense.  Host code only.
//
// "BlockSparseAttention - ComfyUI Built-in Node Documentation", general
// inputs and "constraints and limitations": sequences shorter than
// min_tokens, transformer blocks listed in dense_blocks, and sampling steps
// outside the [start_percent, end_percent] window fall back to dense
// attention; dense_blocks is ignored for a model that reports no block index.
// "minimax-h3-chunk-star7" README, "Hybrid": attention switches between whole
// sampling steps, the guard steps at the front and the back running dense and
// the middle ones sparse (four steps: the first and the fourth dense); without
// a reliable step the run stops with an error.
#include <ctype.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "bsa_internal.h"

namespace bsa {
namespace {

const char *skip_space(const char *s)
{
    while (*s == ' ' || *s == '\t') ++s;
    return s;
}

// Parses a non-negative decimal integer; returns the end or nullptr.
const char *parse_uint(const char *s, long long *out)
{
    if (!isdigit((unsigned char)*s)) return nullptr;
    long long v = 0;
    while (isdigit((unsigned char)*s)) {
        v = v * 10 + (*s - '0');
        if (v > 2147483647LL) return nullptr;
        ++s;
    }
    *out = v;
    return s;
}

}  // namespace

// Whether `block` is listed in `spec` ("0, 1, 47-49": comma-separated
// indices and inclusive ranges, spaces allowed, empty entries ignored).
// Returns 0 / 1, or -1 for a malformed list (message set).
int dense_block_listed(const char *spec, long long block)
{
    if (spec == nullptr) return 0;
    int hit = 0;
    const char *s = spec;
    while (true) {
        s = skip_space(s);
        if (*s == '\0') break;
        if (*s == ',') {
            ++s;
            continue;
        }
        long long a = 0, b = 0;
        const char *e = parse_uint(s, &a);
        if (e == nullptr) {
            set_error("dense_blocks: expected a block index at \"%s\"", s);
            return -1;
        }
        e = skip_space(e);
        b = a;
        if (*e == '-') {
            e = parse_uint(skip_space(e + 1), &b);
            if (e == nullptr || b < a) {
                set_error("dense_blocks: malformed range at \"%s\"", s);
                return -1;
            }
            e = skip_space(e);
        }
        if (*e != ',' && *e != '\0') {
            set_error("dense_blocks: unexpected text at \"%s\"", e);
            return -1;
        }
        if (block >= a && block <= b) hit = 1;
        s = e;
    }
    return hit;
}

}  // namespace bsa

using namespace bsa;

extern "C" {

void bsa_default_policy(bsa_policy *pol)
{
    if (pol == nullptr) return;
    memset(pol, 0, sizeof *pol);
    pol->start_percent = 0.2;
    pol->end_percent = 1.0;
    pol->min_tokens = 12288;
    pol->hybrid = 0;
    pol->hybrid_guard_steps = 1;
    pol->dense_blocks = nullptr;
}

bsa_status bsa_policy_decide(const bsa_policy *pol, int32_t n_tokens, int32_t block_index, double progress,
                             int32_t step, int32_t n_steps, int32_t *decision)
{
    set_error("%s", "");
    if (pol == nullptr || decision == nullptr) {
        set_error("policy / decision is NULL");
        return BSA_ERR_INVALID_ARG;
    }
    if (!(pol->start_percent >= 0.0 && pol->start_percent <= 1.0 && pol->end_percent >= 0.0 &&
          pol->end_percent <= 1.0)) {
        set_error("start_percent and end_percent must lie in [0, 1]");
        return BSA_ERR_INVALID_ARG;
    }
    if (pol->min_tokens < 0) {
        set_error("min_tokens < 0");
        return BSA_ERR_INVALID_ARG;
    }
    if (n_tokens < 1) {
        set_error("n_tokens must be >= 1");
        return BSA_ERR_INVALID_ARG;
    }
    if (!(progress >= 0.0 && progress <= 1.0)) {
        set_error("progress must lie in [0, 1]");
        return BSA_ERR_INVALID_ARG;
    }
    if (pol->hybrid != 0 && pol->hybrid != 1) {
        set_error("hybrid must be 0 or 1");
        return BSA_ERR_INVALID_ARG;
    }
    if (pol->hybrid) {
        if (pol->hybrid_guard_steps < 0) {
            set_error("hybrid_guard_steps < 0");
            return BSA_ERR_INVALID_ARG;
        }
        if (n_steps < 1 || step < 0 || step >= n_steps) {
            set_error("hybrid attention needs the sampling step: step %d of %d cannot be placed", step, n_steps);
            return BSA_ERR_INVALID_ARG;
        }
    }
    // every argument is checked before any decision, so a malformed list is
    // reported whatever the other inputs decide
    int listed = 0;
    if (block_index >= 0) {
        listed = dense_block_listed(pol->dense_blocks, block_index);
        if (listed < 0) return BSA_ERR_INVALID_ARG;
    } else if (dense_block_listed(pol->dense_blocks, 0) < 0) {
        return BSA_ERR_INVALID_ARG;
    }
    if (n_tokens < pol->min_tokens) {
        *decision = BSA_DENSE_SHORT;
    } else if (listed) {
        *decision = BSA_DENSE_BLOCK;
    } else if (pol->hybrid &&
               (step < pol->hybrid_guard_steps || step >= n_steps - pol->hybrid_guard_steps)) {
        *decision = BSA_DENSE_HYBRID;
    } else if (progress < pol->start_percent || progress > pol->end_percent) {
        *decision = BSA_DENSE_WINDOW;
    } else {
        *decision = BSA_RUN_SPARSE;
    }
    return BSA_OK;
}

}  // extern "C"
