// pp_batcher.cpp - host-side batch planning for packed preference groups (pp.h, pp_plan_batches).
//
// "Preference Packing" (abstract and method digest): preference packing combines with batch sorting, and the batch
// size follows the data's lengths to balance compute and memory. A group (one prompt with its responses, packed
// once) costs its packed length; with sorting, groups are taken longest first (a stable sort, so ties keep their
// input order); batches are filled greedily in that order up to a token capacity; a group longer than the
// capacity forms a batch of its own. Plain host code: the plan is made once per epoch over integers.
#include <algorithm>
#include <cstdint>
#include <numeric>
#include <vector>

#include "../../include/pp.h"

extern "C" PP_API pp_status pp_plan_batches(const int64_t *group_tokens, int32_t num_groups, int64_t token_capacity,
                                            int32_t sort_by_length, int32_t *order, int32_t *batch_of_group,
                                            int32_t *num_batches) {
    if (num_groups < 0 || token_capacity < 1 || !num_batches) return PP_ERR_INVALID_ARG;
    if (num_groups > 0 && (!group_tokens || !order || !batch_of_group)) return PP_ERR_INVALID_ARG;
    for (int32_t g = 0; g < num_groups; ++g)
        if (group_tokens[g] < 0) return PP_ERR_INVALID_ARG;
    std::iota(order, order + num_groups, 0);
    if (sort_by_length)
        std::stable_sort(order, order + num_groups,
                         [&](int32_t a, int32_t b) { return group_tokens[a] > group_tokens[b]; });
    int32_t batch = 0;
    int64_t filled = 0, members = 0;
    for (int32_t i = 0; i < num_groups; ++i) {
        const int32_t g = order[i];
        const int64_t t = group_tokens[g];
        if (members > 0 && filled + t > token_capacity) {   // the group does not fit: close the batch
            ++batch;
            filled = 0;
            members = 0;
        }
        batch_of_group[g] = batch;
        filled += t;
        ++members;
    }
    *num_batches = num_groups > 0 ? batch + 1 : 0;
    return PP_OK;
}
