"""B200-native Hyena gated FFT long convolution (package stub; binding added below)."""
