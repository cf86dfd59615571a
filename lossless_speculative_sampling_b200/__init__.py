"""B200-native (sm_100a) Psi-Spec lossless verification: a C-ABI CUDA library (libpsispec.so)
and a thin Python binding over it.

    from lossless_speculative_sampling_b200 import psispec
    tokens, q, stats = psispec.sample_draft(draft_logits, temperature, top_p, u_draft)
    out = psispec.verify_linear(target_logits, draft_logits, tokens, u_accept, u_resid,
                                temperature, top_p, draft_row_stats=stats)

The binding only marshals torch CUDA tensors into the C ABI; every step of the method runs in
the library's kernels. There is no CPU path: without the built library every call raises.
"""
__all__ = ["psispec", "synth"]
