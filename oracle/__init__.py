"""CPU oracle of the TempCache step: TEST INFRASTRUCTURE ONLY.

A plain, slow fp64 implementation written from the FAST-AR pages, used to check
the CUDA path. Only tests/, the package's smoke() check and bench.py's
CPU-baseline leg may import it; the product path never does, and the two share
no code.
"""
from .tempcache_oracle import (  # noqa: F401
    CapacityExceeded,
    CommitRecord,
    OracleTempCache,
    biased_attention,
    cosine_similarity,
    merge_decision,
    seq_dot,
    simhash_codes,
    top1_in_bucket,
)
from .annca_oracle import (  # noqa: F401
    annca_cross_attention,
    kept_prompt_tokens,
)
from .annsa_oracle import (  # noqa: F401
    annsa_attention,
    same_bucket_groups,
)
from .lvsa_oracle import (  # noqa: F401
    attended_frames,
    global_frames,
    local_window,
    lvsa_attention,
)
