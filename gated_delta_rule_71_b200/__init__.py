"""B200-native gated delta rule: chunked forward and GDP decode behind a C ABI."""
