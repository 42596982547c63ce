/* A plain C client of the library's C ABI (host-only entry points).
 *
 * Built with a C compiler against include/muonadamw.h and linked against the
 * shared library, it checks that the header is valid C, that the symbols
 * resolve, and that the host-only entry points behave as documented:
 * ma_partition, ma_assign_owners, ma_shard_layout, ma_status_string,
 * ma_struct_size and the argument checks of muon_workspace_bytes.
 * Prints "ok" and exits 0 on success; prints the failed check and exits 1. */
#include <stdio.h>
#include <string.h>
#include <stdint.h>

#include "muonadamw.h"

static int failures = 0;
#define CHECK(c) do { if (!(c)) { printf("check failed: %s (line %d)\n", #c, __LINE__); ++failures; } } while (0)

static ma_tensor_t tensor(int ndim, int64_t r, int64_t c, int role, int group) {
    ma_tensor_t t;
    memset(&t, 0, sizeof t);
    t.ndim = ndim;
    t.shape[0] = r;
    t.shape[1] = c;
    t.role = role;
    t.group = group;
    return t;
}

int main(void) {
    CHECK(ma_version() == MA_VERSION);
    CHECK(ma_struct_size(0) == sizeof(ma_tensor_t));
    CHECK(ma_struct_size(1) == sizeof(ma_group_t));
    CHECK(ma_struct_size(2) == sizeof(ma_muon_hparams_t));
    CHECK(ma_struct_size(3) == sizeof(ma_adamw_hparams_t));
    CHECK(ma_struct_size(4) == sizeof(ma_shard_slot_t));
    CHECK(ma_struct_size(5) == sizeof(ma_shard_bucket_t));
    CHECK(ma_struct_size(6) == 0);
    CHECK(strlen(ma_status_string(MA_ERR_TIMEOUT)) > 0);

    /* a 2-layer toy model: 4 hidden matrices of two shapes, an embedding, a gain, a scalar */
    ma_tensor_t t[7];
    t[0] = tensor(2, 64, 128, MA_ROLE_EMBED, 1);
    t[1] = tensor(2, 32, 64, MA_ROLE_HIDDEN, 0);
    t[2] = tensor(2, 64, 32, MA_ROLE_HIDDEN, 0);
    t[3] = tensor(2, 32, 64, MA_ROLE_HIDDEN, 0);
    t[4] = tensor(2, 64, 32, MA_ROLE_HIDDEN, 0);
    t[5] = tensor(1, 64, 0, MA_ROLE_HIDDEN, 1);
    t[6] = tensor(0, 0, 0, MA_ROLE_HIDDEN, 1);
    int32_t kind[7];
    CHECK(ma_partition(t, 7, kind) == MA_OK);
    const int32_t want[7] = {MA_ADAMW, MA_MUON, MA_MUON, MA_MUON, MA_MUON, MA_ADAMW, MA_ADAMW};
    for (int i = 0; i < 7; ++i) CHECK(kind[i] == want[i]);

    ma_group_t g[2];
    memset(g, 0, sizeof g);
    g[0].kind = MA_MUON;
    g[0].muon.ns_steps = 5;
    g[0].muon.n_coeffs = 1;
    g[0].muon.heads = 1;
    g[1].kind = MA_ADAMW;

    int32_t owner[7];
    CHECK(ma_assign_owners(t, 7, g, 2, 2, owner) == MA_OK);
    for (int i = 0; i < 7; ++i) CHECK(owner[i] == 0 || owner[i] == 1);
    CHECK(ma_assign_owners(t, 7, g, 2, 0, owner) == MA_ERR_ARG);

    /* two ranks: two full Muon buckets (one per shape), one AdamW bucket */
    ma_shard_slot_t slot[7];
    ma_shard_bucket_t bucket[7];
    int nb = -1;
    int64_t total = -1;
    CHECK(ma_shard_layout(t, 7, g, 2, 2, 1 << 20, slot, bucket, &nb, &total) == MA_OK);
    CHECK(nb == 3);
    CHECK(bucket[0].kind == MA_ADAMW && bucket[1].kind == MA_MUON && bucket[2].kind == MA_MUON);
    CHECK(bucket[1].count == 2 && bucket[1].seg == 32 * 64);
    CHECK(slot[1].owner == 0 && slot[3].owner == 1 && slot[2].owner == 0 && slot[4].owner == 1);
    CHECK(slot[0].owner == -1 && slot[5].owner == -1 && slot[6].owner == -1);
    /* AdamW: 8192 + 64 + 64 elements end to end, split in two segments of 4160 */
    CHECK(bucket[0].start == 0 && bucket[0].seg == 4160);
    CHECK(slot[0].offset == 0 && slot[5].offset == 8192 && slot[6].offset == 8256);
    CHECK(bucket[1].start == 8320 && slot[3].offset == 8320 + 2048);
    CHECK(total == 8320 + 2 * 2048 + 2 * 2048);
    for (int i = 0; i < 7; ++i) CHECK(slot[i].offset % MA_SHARD_ALIGN == 0);
    CHECK(ma_shard_layout(t, 7, g, 2, 2, 0, slot, bucket, &nb, &total) == MA_ERR_ARG);
    CHECK(ma_shard_layout(t, 7, g, 2, 2, 64, NULL, bucket, &nb, &total) == MA_ERR_NULL);

    /* argument checks that need no device */
    ma_muon_hparams_t hp = g[0].muon;
    hp.lr = 0.02f;
    hp.beta = 0.95f;
    hp.coeffs[0][0] = 1.5f;
    hp.coeffs[0][1] = -0.5f;
    CHECK(muon_workspace_bytes(0, 32, 64, &hp) == 0);
    CHECK(muon_workspace_bytes(4, 32, 64, &hp) > 0);
    hp.ns_steps = 0;
    CHECK(muon_workspace_bytes(4, 32, 64, &hp) == (size_t)-1);

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
