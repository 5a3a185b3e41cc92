"""Workload shapes used by the GPU parity tests: the five measured workloads
(some at full size) and reduced versions that the oracle finishes in seconds
while still spanning several tiles and ragged tails."""
from dsa_workloads import CONFIGS

SMALL = {
    "tiny_prefill_1k": CONFIGS["tiny_prefill_1k"],
    "decode_small": CONFIGS["decode_b64_8k_32k"].scaled(name="decode_small", batch=6, ctx=(300, 3000), topk=512,
                                                        planted=16),
    "decode_b4_8k_32k": CONFIGS["decode_b64_8k_32k"].scaled(name="decode_b4_8k_32k", batch=4),
    "prefill_fp8_700": CONFIGS["long_prefill_32k"].scaled(name="prefill_fp8_700", ctx=(700, 700), topk=128,
                                                          heads=32),
    "chunked_small": CONFIGS["chunked_prefill_16"].scaled(name="chunked_small", batch=3, prefix=(0, 3000),
                                                          chunk=(100, 400), topk=256, heads=64),
    "pool_b2_128k": CONFIGS["decode_b8_128k"].scaled(name="pool_b2_128k", batch=2),
}
FULL = dict(CONFIGS)


_cache: dict = {}


def workload(spec):
    """make_workload with a small host-side cache (full-size workloads take seconds to draw)."""
    from dsa_workloads import make_workload
    if spec not in _cache:
        if len(_cache) >= 2:
            _cache.pop(next(iter(_cache)))
        _cache[spec] = make_workload(spec)
    return _cache[spec]
