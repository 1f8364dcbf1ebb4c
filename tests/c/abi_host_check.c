/* A plain C99 user of the library's C ABI (host-only calls, no GPU needed): the header
 * compiles as C, and the partitioner's tables and counters for two small layouts come
 * out as the closed forms say.  Prints "ok" and exits 0, or names the first mismatch. */
#include <stdio.h>
#include <stdlib.h>

#include "zero.h"

static int failures = 0;

static void expect(int cond, const char *what)
{
    if (!cond) {
        printf("FAIL: %s\n", what);
        ++failures;
    }
}

int main(void)
{
    /* the three-GPU walk-through: psi = 3, N = 3, shard rounding 1, one bucket */
    const int64_t one[1] = {3};
    zero_layout_desc d = {3, 1, 1, one, 0, 1, 0, NULL, 0};
    zero_layout *L = NULL;
    zero_layout_info info;
    int64_t toff[1], buckets[2], segs[3 * 4], units[2];
    expect(zero_layout_create(&d, &L) == ZERO_OK && L != NULL, "create walk-through layout");
    expect(zero_layout_get_info(L, &info) == ZERO_OK, "info");
    expect(info.psi == 3 && info.shard == 1 && info.padded == 3, "psi, S, P of the walk-through");
    expect(info.n_buckets == 1 && info.n_segments == 3 && info.n_units == 1, "one bucket, three chunks");
    expect(zero_layout_get_tables(L, toff, buckets, segs, units) == ZERO_OK, "tables");
    expect(buckets[0] == 0 && buckets[1] == 3, "bucket [0, 3)");
    for (int k = 0; k < 3; ++k)
        expect(segs[4 * k] == 0 && segs[4 * k + 1] == k && segs[4 * k + 2] == k && segs[4 * k + 3] == k + 1,
               "chunk k = element k, owned by shard k");
    zero_layout_destroy(L);

    /* ZeRO-3, N = 4: psi = 1031, S = roundup(ceil(1031 / 4), 8) = 264, P = 1056 */
    const int64_t sizes[3] = {1000, 24, 7};
    const int64_t first[2] = {0, 2};
    zero_layout_desc d3 = {4, 3, 3, sizes, 100, 8, 2, first, 0};
    zero_counters c;
    expect(zero_layout_create(&d3, &L) == ZERO_OK, "create ZeRO-3 layout");
    expect(zero_layout_get_info(L, &info) == ZERO_OK, "info");
    expect(info.psi == 1031 && info.shard == 264 && info.padded == 1056, "psi, S, P");
    expect(info.n_buckets == 11 && info.n_units == 2, "11 tail-first buckets, 2 units");
    int64_t b3[2 * 11], u3[2 * 2];
    expect(zero_layout_get_tables(L, NULL, b3, NULL, u3) == ZERO_OK, "tables");
    expect(b3[0] == 956 && b3[1] == 1056 && b3[20] == 0 && b3[21] == 56, "bucket 0 is the tail, the last one the head");
    expect(u3[0] == 0 && u3[1] == 1024 && u3[2] == 1024 && u3[3] == 1056, "units by tensor, the last takes the padding");
    expect(zero_layout_counters(L, &c) == ZERO_OK, "counters");
    expect(c.mem_p16 == 2 * 264 && c.mem_g16 == 2 * 264 && c.mem_os == 12 * 264, "ZeRO-3 shards all three");
    expect(c.sent_elems == 3 * 3 * 264 && c.recv_elems == c.sent_elems, "forward + backward gather + RS");
    zero_layout_destroy(L);

    /* refused descriptions, and every status has a string */
    zero_layout_desc bad = d3;
    bad.stage = 4;
    expect(zero_layout_create(&bad, &L) == ZERO_ERR_INVALID, "stage 4 refused");
    for (int s = ZERO_OK; s <= ZERO_ERR_STATE; ++s)
        expect(zero_status_string((zero_status)s) != NULL, "status string");

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
