"""Block-sparse prefill attention with block-mean correction for B200."""
