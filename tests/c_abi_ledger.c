/* A plain C caller of libzero's host-only calls: the headers must compile as
 * C and the symbols link without C++ or CUDA on the caller's side. Prints the
 * ledger of the 7.5B-parameter, Nd = 64 running example ([P1] stage table),
 * the offloaded step's residency for stage 2, and the peer descriptor's
 * size. */
#include <stdio.h>

#include "zero.h"
#include "zero_offload.h"
#include "zero_peer.h"

int main(void)
{
    zero_config cfg = {0};
    cfg.psi = 7500000000LL;
    cfg.nd = 64;
    cfg.stage = 2;
    cfg.rank_view = 0;
    cfg.variant = ZERO_VARIANT_FUSED;
    zero_ledger L;
    int rc = zero_state_bytes(&cfg, &L);
    if (rc != ZERO_OK) {
        printf("error %d %s\n", rc, zero_error_string(rc));
        return 1;
    }
    printf("formula %.0f %.0f %.0f %.0f\n", L.formula_bytes[0], L.formula_bytes[1], L.formula_bytes[2],
           L.formula_bytes[3]);
    printf("partition %lld\n", (long long)L.partition_len);
    zero_offload_ledger O;
    rc = zero_offload_bytes(&cfg, 0, &O);
    if (rc != ZERO_OK) return 2;
    printf("offload %lld %lld\n", (long long)O.host_state_bytes, (long long)O.device_state_bytes);
    cfg.nd = 0;
    printf("bad %d\n", zero_state_bytes(&cfg, &L));
    zero_peer_desc d = {0};
    printf("peer %u %d\n", (unsigned)sizeof d, zero_peer_open(&d, NULL));
    return 0;
}
