"""Worker for running the oracle's weight quantiser in a spawn process pool
(kept in its own light module so that workers import only the oracle)."""


def quantize_expert(mats):
    from oracle import nvfp4
    return tuple(nvfp4.quantize_weight(m) for m in mats)
